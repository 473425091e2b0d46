// C ABI of the HSTU layer: argument checks, workspace layout, and the
// composition of the step kernels into layer forward / backward /
// M-FALCON cached forward.  See include/hstu.h for the contract.
#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>
#include <atomic>
#include <cstdlib>

#include <nvtx3/nvToolsExt.h>

#include "common.cuh"
#include "internal.h"

using namespace hstu;

namespace {

// ---------------------------------------------------------------------------
// Profiler and launch counter
// ---------------------------------------------------------------------------
struct ProfRecord {
  int id;
  cudaEvent_t start, stop;
};
std::mutex g_prof_mu;
bool g_prof_on = false;
std::vector<ProfRecord> g_prof_records;
std::vector<cudaEvent_t> g_event_pool;
std::vector<std::pair<int, cudaEvent_t>> g_open;  // started, not yet stopped
std::atomic<int64_t> g_launches{0};

// NVTX ranges around the same regions as the profiler's events, named after
// the kernel class, for NVTX-aware tracers; off unless HSTU_NVTX=1 or
// hstu_nvtx_enable(1).
bool nvtx_env() {
  const char* v = std::getenv("HSTU_NVTX");
  return v && v[0] == '1';
}
std::atomic<bool> g_nvtx{nvtx_env()};
const char* const kClassNames[HSTU_K_COUNT] = {
    "proj_in", "attn_fwd", "ln_fwd", "proj_out", "proj_out_bwd", "ln_bwd",
    "attn_bwd", "proj_in_bwd", "attn_cached", "misc", "softmax_fwd"};

cudaEvent_t take_event() {
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

// ---------------------------------------------------------------------------
// Argument checks
// ---------------------------------------------------------------------------
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

hstu_status check_cfg(const hstu_config* c) {
  if (!c) return HSTU_ERR_INVALID;
  if (c->dtype != HSTU_F32 && c->dtype != HSTU_BF16) return HSTU_ERR_INVALID;
  if (c->io_dtype != HSTU_F32 && c->io_dtype != HSTU_BF16) return HSTU_ERR_INVALID;
  if (c->io_dtype != c->dtype && !(c->dtype == HSTU_BF16 && c->io_dtype == HSTU_F32))
    return HSTU_ERR_UNSUPPORTED;
  if (c->d_model <= 0 || c->num_heads <= 0 || c->head_dim <= 0) return HSTU_ERR_INVALID;
  if (c->num_heads * c->head_dim != c->d_model) return HSTU_ERR_INVALID;
  if (!(c->norm_N > 0.f) || !std::isfinite(c->norm_N)) return HSTU_ERR_INVALID;
  if (!(c->ln_eps >= 0.f) || !std::isfinite(c->ln_eps)) return HSTU_ERR_INVALID;
  if (c->max_seq_len <= 0) return HSTU_ERR_INVALID;
  if (c->head_dim != 32 && c->head_dim != 64 && c->head_dim != 128) return HSTU_ERR_UNSUPPORTED;
  if (c->d_model % 16 != 0 || c->d_model > 2048) return HSTU_ERR_UNSUPPORTED;
  if (c->num_pos_buckets < 1 || c->num_pos_buckets > 32) return HSTU_ERR_UNSUPPORTED;
  if (c->num_time_buckets < 1 || c->num_time_buckets > 32) return HSTU_ERR_UNSUPPORTED;
  if (c->max_seq_len > 65536) return HSTU_ERR_UNSUPPORTED;
  return HSTU_OK;
}

// Required pointer: non-null and 16-byte aligned when count > 0.
hstu_status need(const void* p, int64_t count) {
  if (count <= 0) return HSTU_OK;
  if (!p) return HSTU_ERR_INVALID;
  return aligned16(p) ? HSTU_OK : HSTU_ERR_UNSUPPORTED;
}
// Optional pointer: may be null; aligned when present.
hstu_status opt(const void* p) { return (!p || aligned16(p)) ? HSTU_OK : HSTU_ERR_UNSUPPORTED; }
// Metadata pointers (int64/int32 arrays) need natural alignment only.
hstu_status meta(const void* p, int64_t count, size_t align) {
  if (count <= 0) return HSTU_OK;
  if (!p) return HSTU_ERR_INVALID;
  return (reinterpret_cast<uintptr_t>(p) % align) == 0 ? HSTU_OK : HSTU_ERR_UNSUPPORTED;
}

#define HSTU_TRY(x)                         \
  do {                                      \
    hstu_status _s = (x);                   \
    if (_s != HSTU_OK) return _s;           \
  } while (0)
#define HSTU_CUDA(x)                        \
  do {                                      \
    cudaError_t _e = (x);                   \
    if (_e != cudaSuccess) return HSTU_ERR_CUDA; \
  } while (0)

// ---------------------------------------------------------------------------
// Layouts
// ---------------------------------------------------------------------------
void saved_offsets(const hstu_config* c, int64_t T, size_t off[HSTU_SAVED_COUNT + 1]) {
  const size_t es = (size_t)dtype_size(c->dtype);
  const size_t d = (size_t)c->d_model;
  const size_t t = (size_t)T;
  const size_t xlow = c->io_dtype != c->dtype ? t * d * es : 0;
  const size_t sizes[HSTU_SAVED_COUNT] = {t * 4 * d * es, t * 4 * d * es, t * d * 4,
                                          t * d * es,     t * 4,          t * 4, xlow};
  size_t o = 0;
  for (int i = 0; i < HSTU_SAVED_COUNT; ++i) {
    off[i] = o;
    o = align_up(o + sizes[i], 256);
  }
  off[HSTU_SAVED_COUNT] = o;
}

struct FwdWs {
  size_t g, o, z, xlow, attn, total;
};
FwdWs fwd_ws(const hstu_config* c, int B, int64_t T) {
  const size_t es = (size_t)dtype_size(c->dtype), d = (size_t)c->d_model;
  const size_t t = (size_t)T;
  FwdWs w;
  w.g = 0;
  w.o = align_up(w.g + t * 4 * d * es, 256);
  w.z = align_up(w.o + t * d * 4, 256);
  w.xlow = align_up(w.z + t * d * es, 256);
  w.attn = align_up(w.xlow + (c->io_dtype != c->dtype ? t * d * es : 0), 256);
  w.total = align_up(
      w.attn + attention_fwd_ws_full(c->dtype, B, T, c->num_heads, c->head_dim), 256);
  return w;
}

struct BwdWs {
  size_t dz, dO, dpre, dq, dylow, attn, total;
};
BwdWs bwd_ws(const hstu_config* c, int B, int64_t T) {
  const size_t es = (size_t)dtype_size(c->dtype), d = (size_t)c->d_model;
  const size_t t = (size_t)T;
  BwdWs w;
  w.dz = 0;
  w.dO = align_up(w.dz + t * d * es, 256);
  w.dpre = align_up(w.dO + t * d * es, 256);
  w.dq = align_up(w.dpre + t * 4 * d * es, 256);
  w.dylow = align_up(w.dq + t * d * 4, 256);
  w.attn = align_up(w.dylow + (c->io_dtype != c->dtype ? t * d * es : 0), 256);
  w.total = align_up(w.attn + attention_bwd_ws(c->dtype, B, T, c->num_heads, c->head_dim), 256);
  return w;
}

char* at(void* base, size_t off) { return static_cast<char*>(base) + off; }

// ---------------------------------------------------------------------------
// Step implementations (argument checks done by the callers)
// ---------------------------------------------------------------------------
hstu_status do_proj_in(const hstu_config* c, const void* W1, const void* b1, const void* x,
                       int64_t T, void* pre, void* g, cudaStream_t s) {
  const int d = c->d_model;
  GemmArgs a;
  a.A = x; a.lda = d; a.a_kmajor = true;
  a.B = W1; a.ldb = 4 * d; a.b_kmajor = false;
  a.M = T; a.N = 4 * d; a.K = d;
  a.epi = EPI_SILU_SPLIT; a.C = pre; a.C2 = g; a.ldc = 4 * d; a.bias = b1;
  prof_begin(HSTU_K_PROJ_IN, s);
  cudaError_t e = gemm(c->dtype, a, s);
  prof_end(HSTU_K_PROJ_IN, s);
  return e == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}

AttnArgs full_attn_args(const hstu_config* c, const float* rp, const float* rt, const void* g,
                        const int64_t* offs, int B, int64_t T, const int64_t* ts,
                        const int32_t* nt, void* o) {
  const int d = c->d_model, es = dtype_size(c->dtype);
  AttnArgs a;
  a.q = at(const_cast<void*>(g), (size_t)2 * d * es);
  a.self_k = at(const_cast<void*>(g), (size_t)3 * d * es);
  a.self_v = at(const_cast<void*>(g), (size_t)d * es);
  a.q_stride = 4 * d;
  a.k = a.self_k;
  a.v = a.self_v;
  a.kv_stride = 4 * d;
  a.o = o;
  a.o_stride = d;
  a.q_offsets = offs;
  a.kv_offsets = offs;
  a.q_ts = ts;
  a.kv_ts = ts;
  a.num_targets = nt;
  a.cached = 0;
  a.B = B;
  a.H = c->num_heads;
  a.dh = c->head_dim;
  a.P = c->num_pos_buckets;
  a.Bt = c->num_time_buckets;
  a.max_q_len = c->max_seq_len;
  a.q_rows = T;
  a.kv_rows = T;
  a.rab_pos = rp;
  a.rab_time = rt;
  a.inv_N = 1.0f / c->norm_N;
  return a;
}

hstu_status do_attention_fwd(const hstu_config* c, const AttnArgs& a, void* ws, size_t wsb,
                             cudaStream_t s, int prof_id) {
  prof_begin(prof_id, s);
  cudaError_t e = attention_fwd(c->dtype, a, ws, wsb, s);
  prof_end(prof_id, s);
  return e == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}

hstu_status do_ln_fwd(const hstu_config* c, const void* gamma, const void* beta, const void* o,
                      const void* g, int64_t T, void* z, float* mean, float* rstd,
                      cudaStream_t s) {
  prof_begin(HSTU_K_LN_FWD, s);
  cudaError_t e = ln_gate_fwd(c->dtype, c->d_model, c->ln_eps, gamma, beta,
                              static_cast<const float*>(o), g,
                              4 * (int64_t)c->d_model, T, z, mean, rstd, s);
  prof_end(HSTU_K_LN_FWD, s);
  return e == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}

// y_low (bf16, optional): the copy of the fp32 output y that the next layer's
// projection reads, written by the same epilogue (fp32 residual stream only).
hstu_status do_proj_out(const hstu_config* c, const void* W2, const void* b2, const void* z,
                        const void* x, int64_t T, void* y, cudaStream_t s,
                        void* y_low = nullptr) {
  const int d = c->d_model;
  GemmArgs a;
  a.A = z; a.lda = d; a.a_kmajor = true;
  a.B = W2; a.ldb = d; a.b_kmajor = false;
  a.M = T; a.N = d; a.K = d;
  a.epi = x ? EPI_RESID : EPI_STORE; a.C = y; a.ldc = d; a.bias = b2; a.R = x; a.ldr = d;
  a.io_f32 = c->io_dtype == HSTU_F32;
  if (x && a.io_f32 && c->dtype == HSTU_BF16) a.C2 = y_low;
  prof_begin(HSTU_K_PROJ_OUT, s);
  cudaError_t e = gemm(c->dtype, a, s);
  prof_end(HSTU_K_PROJ_OUT, s);
  return e == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}

hstu_status do_proj_out_bwd(const hstu_config* c, const void* W2, const void* z, const void* dy,
                            int64_t T, void* dz, float* dW2, float* db2, cudaStream_t s) {
  const int d = c->d_model;
  prof_begin(HSTU_K_PROJ_OUT_BWD, s);
  GemmArgs a;
  a.A = dy; a.lda = d; a.a_kmajor = true;
  a.B = W2; a.ldb = d; a.b_kmajor = true;
  a.M = T; a.N = d; a.K = d;
  a.epi = EPI_STORE; a.C = dz; a.ldc = d;
  cudaError_t e = gemm(c->dtype, a, s);
  if (e == cudaSuccess && dW2) {
    GemmArgs w;
    w.A = z; w.lda = d; w.a_kmajor = false;
    w.B = dy; w.ldb = d; w.b_kmajor = false;
    w.M = d; w.N = d; w.K = T;
    w.epi = EPI_ATOMIC_F32; w.Cf = dW2; w.ldc = d;
    e = gemm(c->dtype, w, s);
  }
  if (e == cudaSuccess && db2) e = colsum_accumulate(c->dtype, dy, T, d, d, db2, s);
  prof_end(HSTU_K_PROJ_OUT_BWD, s);
  return e == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}

hstu_status do_ln_bwd(const hstu_config* c, const void* gamma, const void* beta, const void* dz,
                      const void* o, const void* g, const void* pre, const float* mean,
                      const float* rstd, int64_t T, void* dO, void* dpre, float* dgamma,
                      float* dbeta, cudaStream_t s) {
  prof_begin(HSTU_K_LN_BWD, s);
  cudaError_t e = ln_gate_bwd(c->dtype, c->d_model, gamma, beta, dz,
                              static_cast<const float*>(o), g, pre,
                              4 * (int64_t)c->d_model, mean, rstd, T, dO, dpre, dgamma, dbeta, s);
  prof_end(HSTU_K_LN_BWD, s);
  return e == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}

hstu_status do_attention_bwd(const hstu_config* c, const float* rp, const float* rt,
                             const void* g, const void* pre, const void* dO, const int64_t* offs,
                             int B, int64_t T, const int64_t* ts, const int32_t* nt, void* dpre,
                             float* drp, float* drt, float* dq_acc, void* ws, size_t wsb,
                             cudaStream_t s) {
  const int d = c->d_model, es = dtype_size(c->dtype);
  AttnBwdArgs a;
  a.f = full_attn_args(c, rp, rt, g, offs, B, T, ts, nt, nullptr);
  a.dout = dO;
  a.pre = pre;
  a.dpre = dpre;
  a.pre_stride = 4 * d;
  a.d = d;
  a.dq_acc = dq_acc;
  a.drab_pos = drp;
  a.drab_time = drt;
  prof_begin(HSTU_K_MISC, s);
  cudaError_t e = T > 0 ? cudaMemsetAsync(dq_acc, 0, (size_t)T * d * 4, s) : cudaSuccess;
  prof_end(HSTU_K_MISC, s);
  if (e != cudaSuccess) return HSTU_ERR_CUDA;
  prof_begin(HSTU_K_ATTN_BWD, s);
  e = attention_bwd(c->dtype, a, ws, wsb, s);
  prof_end(HSTU_K_ATTN_BWD, s);
  if (e != cudaSuccess) return HSTU_ERR_CUDA;
  prof_begin(HSTU_K_MISC, s);
  e = dq_finalize(c->dtype, dq_acc, at(const_cast<void*>(pre), (size_t)2 * d * es), 4 * d,
                  at(dpre, (size_t)2 * d * es), T, d, s);
  prof_end(HSTU_K_MISC, s);
  return e == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}

// dx_low (bf16, optional): the copy of the fp32 dx that the layer below's
// backward reads as its dY operand, written by the same epilogue.
hstu_status do_proj_in_bwd(const hstu_config* c, const void* W1, const void* x, const void* dpre,
                           const void* dy, int64_t T, void* dx, float* dW1, float* db1,
                           cudaStream_t s, void* dx_low = nullptr) {
  const int d = c->d_model;
  prof_begin(HSTU_K_PROJ_IN_BWD, s);
  GemmArgs a;
  a.A = dpre; a.lda = 4 * d; a.a_kmajor = true;
  a.B = W1; a.ldb = 4 * d; a.b_kmajor = true;
  a.M = T; a.N = d; a.K = 4 * d;
  a.epi = dy ? EPI_RESID : EPI_STORE; a.C = dx; a.ldc = d; a.R = dy; a.ldr = d;
  a.io_f32 = c->io_dtype == HSTU_F32;
  if (dy && a.io_f32 && c->dtype == HSTU_BF16) a.C2 = dx_low;
  cudaError_t e = cudaSuccess;
  // dW1 first: dx may alias dy but never x or dpre
  if (dW1) {
    GemmArgs w;
    w.A = x; w.lda = d; w.a_kmajor = false;
    w.B = dpre; w.ldb = 4 * d; w.b_kmajor = false;
    w.M = d; w.N = 4 * d; w.K = T;
    w.epi = EPI_ATOMIC_F32; w.Cf = dW1; w.ldc = 4 * d;
    e = gemm(c->dtype, w, s);
  }
  if (e == cudaSuccess && db1) e = colsum_accumulate(c->dtype, dpre, T, 4 * d, 4 * d, db1, s);
  if (e == cudaSuccess) e = gemm(c->dtype, a, s);
  prof_end(HSTU_K_PROJ_IN_BWD, s);
  return e == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}

// x (io dtype) -> operand dtype copy when the two differ; returns the operand pointer.
hstu_status to_operand(const hstu_config* c, const void* x, int64_t rows, void* low,
                       const void** out, cudaStream_t s) {
  if (c->io_dtype == c->dtype) {
    *out = x;
    return HSTU_OK;
  }
  prof_begin(HSTU_K_MISC, s);
  cudaError_t e = convert_f32_to_bf16(static_cast<const float*>(x), low, rows * c->d_model, s);
  prof_end(HSTU_K_MISC, s);
  *out = low;
  return e == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}

hstu_status check_jagged(const int64_t* offs, int32_t B, int64_t T, const int64_t* ts,
                         const int32_t* nt) {
  if (B < 0 || T < 0) return HSTU_ERR_INVALID;
  HSTU_TRY(meta(offs, (int64_t)B + 1, 8));
  HSTU_TRY(meta(ts, T, 8));
  if (nt) HSTU_TRY(meta(nt, B, 4));
  return HSTU_OK;
}

hstu_status check_weights(const hstu_config* c, const hstu_weights* w, bool need_w1,
                          bool need_w2) {
  if (!w) return HSTU_ERR_INVALID;
  if (need_w1) HSTU_TRY(need(w->W1, 1));
  if (need_w2) HSTU_TRY(need(w->W2, 1));
  HSTU_TRY(opt(w->b1));
  HSTU_TRY(opt(w->b2));
  HSTU_TRY(opt(w->ln_gamma));
  HSTU_TRY(opt(w->ln_beta));
  HSTU_TRY(meta(w->rab_pos, w->rab_pos ? 1 : 0, 4));
  HSTU_TRY(meta(w->rab_time, w->rab_time ? 1 : 0, 4));
  (void)c;
  return HSTU_OK;
}

}  // namespace

namespace hstu {

// Status word written by device code (bounded waits that ran out).
__device__ uint32_t g_device_status;

uint32_t* device_status() {
  static uint32_t* ptrs[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  if (!ptrs[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
    ptrs[dev] = static_cast<uint32_t*>(p);
  }
  return ptrs[dev];
}

void prof_begin(int id, cudaStream_t s) {
  if (g_nvtx.load(std::memory_order_relaxed) && id >= 0 && id < HSTU_K_COUNT)
    nvtxRangePushA(kClassNames[id]);
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (!g_prof_on) return;
  cudaEvent_t e = take_event();
  if (!e) return;
  cudaEventRecord(e, s);
  g_open.push_back({id, e});
}

void prof_end(int id, cudaStream_t s) {
  if (g_nvtx.load(std::memory_order_relaxed) && id >= 0 && id < HSTU_K_COUNT) nvtxRangePop();
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (!g_prof_on) return;
  for (size_t i = g_open.size(); i-- > 0;) {
    if (g_open[i].first == id) {
      cudaEvent_t e = take_event();
      if (!e) return;
      cudaEventRecord(e, s);
      g_prof_records.push_back({id, g_open[i].second, e});
      g_open.erase(g_open.begin() + (long)i);
      return;
    }
  }
}

void count_launch(int n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

}  // namespace hstu

extern "C" {

const char* hstu_status_string(hstu_status s) {
  switch (s) {
    case HSTU_OK: return "ok";
    case HSTU_ERR_INVALID: return "invalid argument";
    case HSTU_ERR_UNSUPPORTED: return "unsupported shape, dtype or alignment";
    case HSTU_ERR_CUDA: return "CUDA error";
    case HSTU_ERR_WORKSPACE: return "workspace too small";
    case HSTU_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case HSTU_ERR_BAD_INPUT_DATA: return "malformed input data";
  }
  return "unknown status";
}

const char* hstu_version(void) { return "hstu-b200 0.1 (sm_100a)"; }

void hstu_nvtx_enable(int32_t on) { g_nvtx.store(on != 0, std::memory_order_relaxed); }

void hstu_profiler_enable(int32_t on) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_prof_on = on != 0;
}

void hstu_profiler_reset(void) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (auto& r : g_prof_records) {
    g_event_pool.push_back(r.start);
    g_event_pool.push_back(r.stop);
  }
  g_prof_records.clear();
  for (auto& o : g_open) g_event_pool.push_back(o.second);
  g_open.clear();
  g_launches.store(0);
}

hstu_status hstu_profiler_collect(int32_t id, int64_t* launches, double* total_ms) {
  if (!launches || !total_ms) return HSTU_ERR_INVALID;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  int64_t n = 0;
  double ms = 0.0;
  for (auto& r : g_prof_records) {
    if (r.id != id) continue;
    if (cudaEventSynchronize(r.stop) != cudaSuccess) return HSTU_ERR_CUDA;
    float t = 0.f;
    if (cudaEventElapsedTime(&t, r.start, r.stop) != cudaSuccess) return HSTU_ERR_CUDA;
    ms += t;
    ++n;
  }
  *launches = n;
  *total_ms = ms;
  return HSTU_OK;
}

int64_t hstu_launch_count(void) { return g_launches.load(); }

hstu_status hstu_device_status(uint32_t* host_out, int32_t clear, cudaStream_t stream) {
  if (!host_out) return HSTU_ERR_INVALID;
  uint32_t* d = device_status();
  if (!d) return HSTU_ERR_CUDA;
  if (cudaMemcpyAsync(host_out, d, sizeof(uint32_t), cudaMemcpyDeviceToHost, stream) != cudaSuccess)
    return HSTU_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return HSTU_ERR_CUDA;
  if (clear && cudaMemsetAsync(d, 0, sizeof(uint32_t), stream) != cudaSuccess) return HSTU_ERR_CUDA;
  return HSTU_OK;
}

hstu_status hstu_saved_layout(const hstu_config* cfg, int64_t T,
                              size_t offsets[HSTU_SAVED_COUNT + 1]) {
  HSTU_TRY(check_cfg(cfg));
  if (T < 0 || !offsets) return HSTU_ERR_INVALID;
  saved_offsets(cfg, T, offsets);
  return HSTU_OK;
}

size_t hstu_attention_workspace_size(const hstu_config* cfg, int32_t B, int64_t T) {
  if (check_cfg(cfg) != HSTU_OK || B < 0 || T < 0) return 0;
  return attention_fwd_ws_full(cfg->dtype, B, T, cfg->num_heads, cfg->head_dim);
}

size_t hstu_attention_bwd_workspace_size(const hstu_config* cfg, int32_t B, int64_t T) {
  if (check_cfg(cfg) != HSTU_OK || B < 0 || T < 0) return 0;
  return align_up(attention_bwd_ws(cfg->dtype, B, T, cfg->num_heads, cfg->head_dim), 256) +
         align_up((size_t)T * cfg->d_model * 4, 256);
}

hstu_status hstu_workspace_size(const hstu_config* cfg, int32_t B, int64_t T, size_t* ws_bytes,
                                size_t* saved_bytes) {
  HSTU_TRY(check_cfg(cfg));
  if (B < 0 || T < 0) return HSTU_ERR_INVALID;
  if (ws_bytes) {
    size_t f = fwd_ws(cfg, B, T).total, b = bwd_ws(cfg, B, T).total;
    *ws_bytes = f > b ? f : b;
  }
  if (saved_bytes) {
    size_t off[HSTU_SAVED_COUNT + 1];
    saved_offsets(cfg, T, off);
    *saved_bytes = off[HSTU_SAVED_COUNT];
  }
  return HSTU_OK;
}

hstu_status hstu_validate_inputs(const int64_t* seq_offsets, int32_t B, int64_t T,
                                 const int64_t* timestamps, const int32_t* num_targets,
                                 int32_t max_seq_len, uint32_t* d_flags, cudaStream_t stream) {
  HSTU_TRY(check_jagged(seq_offsets, B, T, timestamps, num_targets));
  HSTU_TRY(meta(d_flags, 1, 4));
  prof_begin(HSTU_K_MISC, stream);
  cudaError_t e = validate_inputs(seq_offsets, B, T, timestamps, num_targets, max_seq_len, d_flags,
                                  stream);
  prof_end(HSTU_K_MISC, stream);
  return e == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}

// ----------------------------- step level ---------------------------------

hstu_status hstu_proj_in_fwd(const hstu_config* cfg, const hstu_weights* w, const void* x,
                             int64_t T, void* pre_out, void* g_out, cudaStream_t stream) {
  HSTU_TRY(check_cfg(cfg));
  if (T < 0) return HSTU_ERR_INVALID;
  HSTU_TRY(check_weights(cfg, w, true, false));
  HSTU_TRY(need(x, T));
  HSTU_TRY(need(g_out, T));
  HSTU_TRY(opt(pre_out));
  if (T == 0) return HSTU_OK;
  return do_proj_in(cfg, w->W1, w->b1, x, T, pre_out, g_out, stream);
}

hstu_status hstu_attention_fwd(const hstu_config* cfg, const float* rab_pos, const float* rab_time,
                               const void* g, const int64_t* seq_offsets, int32_t B, int64_t T,
                               const int64_t* timestamps, const int32_t* num_targets, void* o_out,
                               void* workspace, size_t ws_bytes, cudaStream_t stream) {
  HSTU_TRY(check_cfg(cfg));
  HSTU_TRY(check_jagged(seq_offsets, B, T, timestamps, num_targets));
  HSTU_TRY(need(g, T));
  HSTU_TRY(need(o_out, T));
  HSTU_TRY(meta(rab_pos, rab_pos ? 1 : 0, 4));
  HSTU_TRY(meta(rab_time, rab_time ? 1 : 0, 4));
  const size_t need_ws = attention_fwd_ws(B, T, cfg->num_heads);
  if (ws_bytes < need_ws) return HSTU_ERR_WORKSPACE;
  if (need_ws > 0) HSTU_TRY(need(workspace, 1));
  if (T == 0 || B == 0) return HSTU_OK;
  AttnArgs a = full_attn_args(cfg, rab_pos, rab_time, g, seq_offsets, B, T, timestamps,
                              num_targets, o_out);
  return do_attention_fwd(cfg, a, workspace, ws_bytes, stream, HSTU_K_ATTN_FWD);
}

hstu_status hstu_softmax_attention_fwd(const hstu_config* cfg, const float* rab_pos,
                                       const float* rab_time, const void* g,
                                       const int64_t* seq_offsets, int32_t B, int64_t T,
                                       const int64_t* timestamps, const int32_t* num_targets,
                                       void* o_out, void* workspace, size_t ws_bytes,
                                       cudaStream_t stream) {
  HSTU_TRY(check_cfg(cfg));
  HSTU_TRY(check_jagged(seq_offsets, B, T, timestamps, num_targets));
  HSTU_TRY(need(g, T));
  HSTU_TRY(need(o_out, T));
  HSTU_TRY(meta(rab_pos, rab_pos ? 1 : 0, 4));
  HSTU_TRY(meta(rab_time, rab_time ? 1 : 0, 4));
  const size_t need_ws = attention_fwd_ws(B, T, cfg->num_heads);
  if (ws_bytes < need_ws) return HSTU_ERR_WORKSPACE;
  if (need_ws > 0) HSTU_TRY(need(workspace, 1));
  if (T == 0 || B == 0) return HSTU_OK;
  AttnArgs a = full_attn_args(cfg, rab_pos, rab_time, g, seq_offsets, B, T, timestamps,
                              num_targets, o_out);
  if (!softmax_fwd_tc_supported(cfg->dtype, a)) return HSTU_ERR_UNSUPPORTED;
  prof_begin(HSTU_K_SOFTMAX, stream);
  cudaError_t e = softmax_fwd_tc(a, workspace, device_status(), stream);
  prof_end(HSTU_K_SOFTMAX, stream);
  return e == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}

hstu_status hstu_attention_fwd_cached(const hstu_config* cfg, const float* rab_pos,
                                      const float* rab_time, const void* cand_g,
                                      const int64_t* cand_offsets, int32_t B, int64_t Tc,
                                      const int64_t* cand_timestamps, const void* hist_kv,
                                      const int64_t* hist_offsets, int64_t T_hist,
                                      const int64_t* hist_timestamps, void* o_out,
                                      void* workspace, size_t ws_bytes, cudaStream_t stream) {
  HSTU_TRY(check_cfg(cfg));
  HSTU_TRY(check_jagged(cand_offsets, B, Tc, cand_timestamps, nullptr));
  HSTU_TRY(check_jagged(hist_offsets, B, T_hist, hist_timestamps, nullptr));
  HSTU_TRY(need(cand_g, Tc));
  HSTU_TRY(need(hist_kv, T_hist));
  HSTU_TRY(need(o_out, Tc));
  HSTU_TRY(meta(rab_pos, rab_pos ? 1 : 0, 4));
  HSTU_TRY(meta(rab_time, rab_time ? 1 : 0, 4));
  const size_t need_ws = attention_fwd_ws(B, Tc, cfg->num_heads);
  if (ws_bytes < need_ws) return HSTU_ERR_WORKSPACE;
  if (need_ws > 0) HSTU_TRY(need(workspace, 1));
  if (Tc == 0 || B == 0) return HSTU_OK;
  const int d = cfg->d_model, es = dtype_size(cfg->dtype);
  AttnArgs a = full_attn_args(cfg, rab_pos, rab_time, cand_g, cand_offsets, B, Tc,
                              cand_timestamps, nullptr, o_out);
  a.cached = 1;
  a.kv_rows = T_hist;
  a.v = hist_kv;
  a.k = at(const_cast<void*>(hist_kv), (size_t)d * es);
  a.kv_stride = 2 * d;
  a.kv_offsets = hist_offsets;
  a.kv_ts = hist_timestamps;
  return do_attention_fwd(cfg, a, workspace, ws_bytes, stream, HSTU_K_ATTN_CACHED);
}

hstu_status hstu_ln_gate_fwd(const hstu_config* cfg, const void* ln_gamma, const void* ln_beta,
                             const void* o, const void* g, int64_t T, void* z_out, float* mean_out,
                             float* rstd_out, cudaStream_t stream) {
  HSTU_TRY(check_cfg(cfg));
  if (T < 0) return HSTU_ERR_INVALID;
  HSTU_TRY(opt(ln_gamma));
  HSTU_TRY(opt(ln_beta));
  HSTU_TRY(need(o, T));
  HSTU_TRY(need(g, T));
  HSTU_TRY(need(z_out, T));
  HSTU_TRY(meta(mean_out, mean_out ? 1 : 0, 4));
  HSTU_TRY(meta(rstd_out, rstd_out ? 1 : 0, 4));
  if (T == 0) return HSTU_OK;
  return do_ln_fwd(cfg, ln_gamma, ln_beta, o, g, T, z_out, mean_out, rstd_out, stream);
}

hstu_status hstu_proj_out_fwd(const hstu_config* cfg, const void* W2, const void* b2,
                              const void* z, const void* x, int64_t T, void* y_out,
                              cudaStream_t stream) {
  HSTU_TRY(check_cfg(cfg));
  if (T < 0) return HSTU_ERR_INVALID;
  HSTU_TRY(need(W2, 1));
  HSTU_TRY(opt(b2));
  HSTU_TRY(need(z, T));
  HSTU_TRY(opt(x));
  HSTU_TRY(need(y_out, T));
  if (T == 0) return HSTU_OK;
  return do_proj_out(cfg, W2, b2, z, x, T, y_out, stream);
}

hstu_status hstu_proj_out_bwd(const hstu_config* cfg, const void* W2, const void* z,
                              const void* dy, int64_t T, void* dz_out, float* dW2, float* db2,
                              cudaStream_t stream) {
  HSTU_TRY(check_cfg(cfg));
  if (T < 0) return HSTU_ERR_INVALID;
  HSTU_TRY(need(W2, 1));
  HSTU_TRY(need(dy, T));
  HSTU_TRY(need(dz_out, T));
  if (dW2) HSTU_TRY(need(z, T));
  HSTU_TRY(meta(dW2, dW2 ? 1 : 0, 4));
  HSTU_TRY(meta(db2, db2 ? 1 : 0, 4));
  if (T == 0) return HSTU_OK;
  return do_proj_out_bwd(cfg, W2, z, dy, T, dz_out, dW2, db2, stream);
}

hstu_status hstu_ln_gate_bwd(const hstu_config* cfg, const void* ln_gamma, const void* ln_beta,
                             const void* dz, const void* o, const void* g, const void* pre,
                             const float* mean, const float* rstd, int64_t T, void* do_out,
                             void* dpre, float* dgamma, float* dbeta, cudaStream_t stream) {
  HSTU_TRY(check_cfg(cfg));
  if (T < 0) return HSTU_ERR_INVALID;
  HSTU_TRY(opt(ln_gamma));
  HSTU_TRY(opt(ln_beta));
  HSTU_TRY(need(dz, T));
  HSTU_TRY(need(o, T));
  HSTU_TRY(need(g, T));
  HSTU_TRY(need(pre, T));
  HSTU_TRY(meta(mean, T, 4));
  HSTU_TRY(meta(rstd, T, 4));
  HSTU_TRY(need(do_out, T));
  HSTU_TRY(need(dpre, T));
  HSTU_TRY(meta(dgamma, dgamma ? 1 : 0, 4));
  HSTU_TRY(meta(dbeta, dbeta ? 1 : 0, 4));
  if (T == 0) return HSTU_OK;
  return do_ln_bwd(cfg, ln_gamma, ln_beta, dz, o, g, pre, mean, rstd, T, do_out, dpre, dgamma,
                   dbeta, stream);
}

hstu_status hstu_attention_bwd(const hstu_config* cfg, const float* rab_pos,
                               const float* rab_time, const void* g, const void* pre,
                               const void* dout, const int64_t* seq_offsets, int32_t B, int64_t T,
                               const int64_t* timestamps, const int32_t* num_targets, void* dpre,
                               float* drab_pos, float* drab_time, void* workspace,
                               size_t ws_bytes, cudaStream_t stream) {
  HSTU_TRY(check_cfg(cfg));
  HSTU_TRY(check_jagged(seq_offsets, B, T, timestamps, num_targets));
  HSTU_TRY(need(g, T));
  HSTU_TRY(need(pre, T));
  HSTU_TRY(need(dout, T));
  HSTU_TRY(need(dpre, T));
  HSTU_TRY(meta(rab_pos, rab_pos ? 1 : 0, 4));
  HSTU_TRY(meta(rab_time, rab_time ? 1 : 0, 4));
  HSTU_TRY(meta(drab_pos, drab_pos ? 1 : 0, 4));
  HSTU_TRY(meta(drab_time, drab_time ? 1 : 0, 4));
  const size_t attn = align_up(attention_bwd_ws(cfg->dtype, B, T, cfg->num_heads,
                                                cfg->head_dim), 256);
  if (ws_bytes < hstu_attention_bwd_workspace_size(cfg, B, T)) return HSTU_ERR_WORKSPACE;
  if (T == 0 || B == 0) return HSTU_OK;
  HSTU_TRY(need(workspace, 1));
  float* dq = reinterpret_cast<float*>(at(workspace, attn));
  return do_attention_bwd(cfg, rab_pos, rab_time, g, pre, dout, seq_offsets, B, T, timestamps,
                          num_targets, dpre, drab_pos, drab_time, dq, workspace, attn, stream);
}

hstu_status hstu_proj_in_bwd(const hstu_config* cfg, const void* W1, const void* x,
                             const void* dpre, const void* dy_resid, int64_t T, void* dx_out,
                             float* dW1, float* db1, cudaStream_t stream) {
  HSTU_TRY(check_cfg(cfg));
  if (T < 0) return HSTU_ERR_INVALID;
  HSTU_TRY(need(W1, 1));
  HSTU_TRY(need(dpre, T));
  HSTU_TRY(opt(dy_resid));
  HSTU_TRY(need(dx_out, T));
  if (dW1) HSTU_TRY(need(x, T));
  HSTU_TRY(meta(dW1, dW1 ? 1 : 0, 4));
  HSTU_TRY(meta(db1, db1 ? 1 : 0, 4));
  if (T == 0) return HSTU_OK;
  return do_proj_in_bwd(cfg, W1, x, dpre, dy_resid, T, dx_out, dW1, db1, stream);
}

// ----------------------------- layer level --------------------------------

hstu_status hstu_fwd(const hstu_config* cfg, const hstu_weights* w, const void* x,
                     const int64_t* seq_offsets, int32_t B, int64_t T, const int64_t* timestamps,
                     const int32_t* num_targets, void* y, void* saved, void* kv_out,
                     void* workspace, size_t ws_bytes, cudaStream_t stream) {
  return hstu_fwd_chain(cfg, w, x, nullptr, seq_offsets, B, T, timestamps, num_targets, y,
                        nullptr, saved, kv_out, workspace, ws_bytes, stream);
}

hstu_status hstu_fwd_chain(const hstu_config* cfg, const hstu_weights* w, const void* x,
                           const void* x_low, const int64_t* seq_offsets, int32_t B, int64_t T,
                           const int64_t* timestamps, const int32_t* num_targets, void* y,
                           void* y_low, void* saved, void* kv_out, void* workspace,
                           size_t ws_bytes, cudaStream_t stream) {
  HSTU_TRY(check_cfg(cfg));
  HSTU_TRY(check_jagged(seq_offsets, B, T, timestamps, num_targets));
  HSTU_TRY(check_weights(cfg, w, true, true));
  HSTU_TRY(need(x, T));
  HSTU_TRY(need(y, T));
  HSTU_TRY(opt(saved));
  HSTU_TRY(opt(kv_out));
  HSTU_TRY(opt(x_low));
  HSTU_TRY(opt(y_low));
  const bool lowio = cfg->io_dtype != cfg->dtype;   // fp32 residual stream, bf16 operands
  if (!lowio) x_low = y_low = nullptr;
  const FwdWs L = fwd_ws(cfg, B, T);
  if (ws_bytes < L.total) return HSTU_ERR_WORKSPACE;
  if (T == 0 || B == 0) return HSTU_OK;
  HSTU_TRY(need(workspace, 1));
  const int d = cfg->d_model, es = dtype_size(cfg->dtype);
  void *pre = nullptr, *g, *o, *z, *xlow = at(workspace, L.xlow);
  float *mean = nullptr, *rstd = nullptr;
  if (saved) {
    size_t off[HSTU_SAVED_COUNT + 1];
    saved_offsets(cfg, T, off);
    pre = at(saved, off[HSTU_SAVED_PRE]);
    g = at(saved, off[HSTU_SAVED_G]);
    o = at(saved, off[HSTU_SAVED_O]);
    z = at(saved, off[HSTU_SAVED_Z]);
    mean = reinterpret_cast<float*>(at(saved, off[HSTU_SAVED_MEAN]));
    rstd = reinterpret_cast<float*>(at(saved, off[HSTU_SAVED_RSTD]));
    xlow = at(saved, off[HSTU_SAVED_XLOW]);
  } else {
    g = at(workspace, L.g);
    o = at(workspace, L.o);
    z = at(workspace, L.z);
  }
  const void* xop = nullptr;
  if (x_low) {
    // the bf16 copy of x came with the call; the saved block keeps its own
    // copy for the backward unless x_low already is that part of it
    xop = x_low;
    if (saved && x_low != xlow) {
      prof_begin(HSTU_K_MISC, stream);
      cudaError_t e = cudaMemcpyAsync(xlow, x_low, (size_t)T * d * es, cudaMemcpyDeviceToDevice,
                                      stream);
      prof_end(HSTU_K_MISC, stream);
      if (e != cudaSuccess) return HSTU_ERR_CUDA;
    }
  } else {
    HSTU_TRY(to_operand(cfg, x, T, xlow, &xop, stream));
  }
  HSTU_TRY(do_proj_in(cfg, w->W1, w->b1, xop, T, pre, g, stream));
  AttnArgs a = full_attn_args(cfg, w->rab_pos, w->rab_time, g, seq_offsets, B, T, timestamps,
                              num_targets, o);
  HSTU_TRY(do_attention_fwd(cfg, a, at(workspace, L.attn), ws_bytes - L.attn, stream,
                            HSTU_K_ATTN_FWD));
  HSTU_TRY(do_ln_fwd(cfg, w->ln_gamma, w->ln_beta, o, g, T, z, mean, rstd, stream));
  HSTU_TRY(do_proj_out(cfg, w->W2, w->b2, z, x, T, y, stream, y_low));
  if (kv_out) {
    prof_begin(HSTU_K_MISC, stream);
    cudaError_t e = copy_columns(cfg->dtype, at(g, (size_t)d * es), 4 * d, kv_out, 2 * d, T, d,
                                 stream);
    if (e == cudaSuccess)
      e = copy_columns(cfg->dtype, at(g, (size_t)3 * d * es), 4 * d, at(kv_out, (size_t)d * es),
                       2 * d, T, d, stream);
    prof_end(HSTU_K_MISC, stream);
    if (e != cudaSuccess) return HSTU_ERR_CUDA;
  }
  return HSTU_OK;
}

hstu_status hstu_fwd_cached(const hstu_config* cfg, const hstu_weights* w, const void* cand_x,
                            const int64_t* cand_offsets, int32_t B, int64_t Tc,
                            const int64_t* cand_timestamps, const void* hist_kv,
                            const int64_t* hist_offsets, int64_t T_hist,
                            const int64_t* hist_timestamps, void* y, void* workspace,
                            size_t ws_bytes, cudaStream_t stream) {
  HSTU_TRY(check_cfg(cfg));
  HSTU_TRY(check_jagged(cand_offsets, B, Tc, cand_timestamps, nullptr));
  HSTU_TRY(check_jagged(hist_offsets, B, T_hist, hist_timestamps, nullptr));
  HSTU_TRY(check_weights(cfg, w, true, true));
  HSTU_TRY(need(cand_x, Tc));
  HSTU_TRY(need(hist_kv, T_hist));
  HSTU_TRY(need(y, Tc));
  const FwdWs L = fwd_ws(cfg, B, Tc);
  if (ws_bytes < L.total) return HSTU_ERR_WORKSPACE;
  if (Tc == 0 || B == 0) return HSTU_OK;
  HSTU_TRY(need(workspace, 1));
  const int d = cfg->d_model, es = dtype_size(cfg->dtype);
  void* g = at(workspace, L.g);
  void* o = at(workspace, L.o);
  void* z = at(workspace, L.z);
  const void* xop = nullptr;
  HSTU_TRY(to_operand(cfg, cand_x, Tc, at(workspace, L.xlow), &xop, stream));
  HSTU_TRY(do_proj_in(cfg, w->W1, w->b1, xop, Tc, nullptr, g, stream));
  AttnArgs a = full_attn_args(cfg, w->rab_pos, w->rab_time, g, cand_offsets, B, Tc,
                              cand_timestamps, nullptr, o);
  a.cached = 1;
  a.kv_rows = T_hist;
  a.v = hist_kv;
  a.k = at(const_cast<void*>(hist_kv), (size_t)d * es);
  a.kv_stride = 2 * d;
  a.kv_offsets = hist_offsets;
  a.kv_ts = hist_timestamps;
  HSTU_TRY(do_attention_fwd(cfg, a, at(workspace, L.attn), ws_bytes - L.attn, stream,
                            HSTU_K_ATTN_CACHED));
  HSTU_TRY(do_ln_fwd(cfg, w->ln_gamma, w->ln_beta, o, g, Tc, z, nullptr, nullptr, stream));
  HSTU_TRY(do_proj_out(cfg, w->W2, w->b2, z, cand_x, Tc, y, stream));
  return HSTU_OK;
}

hstu_status hstu_bwd(const hstu_config* cfg, const hstu_weights* w, const void* x, const void* dy,
                     const void* saved, const int64_t* seq_offsets, int32_t B, int64_t T,
                     const int64_t* timestamps, const int32_t* num_targets, void* dx,
                     const hstu_grads* grads, void* workspace, size_t ws_bytes,
                     cudaStream_t stream) {
  return hstu_bwd_chain(cfg, w, x, dy, nullptr, saved, seq_offsets, B, T, timestamps,
                        num_targets, dx, nullptr, grads, workspace, ws_bytes, stream);
}

hstu_status hstu_bwd_chain(const hstu_config* cfg, const hstu_weights* w, const void* x,
                           const void* dy, const void* dy_low, const void* saved,
                           const int64_t* seq_offsets, int32_t B, int64_t T,
                           const int64_t* timestamps, const int32_t* num_targets, void* dx,
                           void* dx_low, const hstu_grads* grads, void* workspace,
                           size_t ws_bytes, cudaStream_t stream) {
  HSTU_TRY(check_cfg(cfg));
  HSTU_TRY(check_jagged(seq_offsets, B, T, timestamps, num_targets));
  HSTU_TRY(check_weights(cfg, w, true, true));
  HSTU_TRY(opt(dy_low));
  HSTU_TRY(opt(dx_low));
  if (cfg->io_dtype == cfg->dtype) dy_low = dx_low = nullptr;
  HSTU_TRY(need(x, T));
  HSTU_TRY(need(dy, T));
  HSTU_TRY(need(saved, T));
  HSTU_TRY(need(dx, T));
  hstu_grads gr;
  std::memset(&gr, 0, sizeof(gr));
  if (grads) gr = *grads;
  HSTU_TRY(meta(gr.dW1, gr.dW1 ? 1 : 0, 4));
  HSTU_TRY(meta(gr.dW2, gr.dW2 ? 1 : 0, 4));
  const BwdWs L = bwd_ws(cfg, B, T);
  if (ws_bytes < L.total) return HSTU_ERR_WORKSPACE;
  if (T == 0 || B == 0) return HSTU_OK;
  HSTU_TRY(need(workspace, 1));
  size_t off[HSTU_SAVED_COUNT + 1];
  saved_offsets(cfg, T, off);
  void* svd = const_cast<void*>(saved);
  const void* pre = at(svd, off[HSTU_SAVED_PRE]);
  const void* g = at(svd, off[HSTU_SAVED_G]);
  const void* o = at(svd, off[HSTU_SAVED_O]);
  const void* z = at(svd, off[HSTU_SAVED_Z]);
  const float* mean = reinterpret_cast<const float*>(at(svd, off[HSTU_SAVED_MEAN]));
  const float* rstd = reinterpret_cast<const float*>(at(svd, off[HSTU_SAVED_RSTD]));
  void* dz = at(workspace, L.dz);
  void* dO = at(workspace, L.dO);
  void* dpre = at(workspace, L.dpre);
  float* dq = reinterpret_cast<float*>(at(workspace, L.dq));
  const void* xop = cfg->io_dtype == cfg->dtype ? x : at(svd, off[HSTU_SAVED_XLOW]);
  const void* dyop = dy_low;
  if (!dyop) HSTU_TRY(to_operand(cfg, dy, T, at(workspace, L.dylow), &dyop, stream));
  HSTU_TRY(do_proj_out_bwd(cfg, w->W2, z, dyop, T, dz, gr.dW2, gr.db2, stream));
  HSTU_TRY(do_ln_bwd(cfg, w->ln_gamma, w->ln_beta, dz, o, g, pre, mean, rstd, T, dO, dpre,
                     gr.dgamma, gr.dbeta, stream));
  HSTU_TRY(do_attention_bwd(cfg, w->rab_pos, w->rab_time, g, pre, dO, seq_offsets, B, T,
                            timestamps, num_targets, dpre, gr.drab_pos, gr.drab_time, dq,
                            at(workspace, L.attn), ws_bytes - L.attn, stream));
  HSTU_TRY(do_proj_in_bwd(cfg, w->W1, xop, dpre, dy, T, dx, gr.dW1, gr.db1, stream, dx_low));
  return HSTU_OK;
}

}  // extern "C"
