// C ABI of libhla: argument checks, workspace and cache layout, launch sequence.
// Every entry point validates on the host first and launches nothing on error.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include <cuda.h>

#include "common.cuh"
#include "kernels.cuh"

namespace {

thread_local char g_msg[512] = "";

hla_status fail(hla_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return s;
}

hla_status cuda_fail(cudaError_t e, const char* where) {
  return fail(HLA_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

size_t esize(int dtype) { return dtype == HLA_BF16 ? 2 : 4; }

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

// Shape/dtype checks common to every entry point.  need_T: T must be >= 1.
hla_status check_cfg(const hla_config* c, bool need_T) {
  if (c == nullptr) return fail(HLA_ERR_INVALID_ARG, "cfg is NULL");
  if (c->B <= 0 || c->H <= 0) return fail(HLA_ERR_INVALID_ARG, "B and H must be positive (B=%d H=%d)", c->B, c->H);
  if (need_T && c->T <= 0) return fail(HLA_ERR_INVALID_ARG, "T must be positive (T=%d)", c->T);
  if (c->C != 64 && c->C != 128 && c->C != 256)
    return fail(HLA_ERR_UNSUPPORTED, "chunk size C=%d unsupported (64, 128, 256)", c->C);
  if (c->dk != c->dv) return fail(HLA_ERR_UNSUPPORTED, "dk != dv (%d, %d) unsupported", c->dk, c->dv);
  if (c->dk != 64 && c->dk != 128) return fail(HLA_ERR_UNSUPPORTED, "head dim %d unsupported (64, 128)", c->dk);
  if (c->dtype != HLA_F32 && c->dtype != HLA_BF16) return fail(HLA_ERR_UNSUPPORTED, "dtype %d unsupported", c->dtype);
  if (c->gate_mode < HLA_GATES_ROUTED || c->gate_mode > HLA_GATES_USER)
    return fail(HLA_ERR_INVALID_ARG, "gate_mode %d invalid", c->gate_mode);
  if (c->cache_format != HLA_CACHE_DENSE && c->cache_format != HLA_CACHE_FACTORED)
    return fail(HLA_ERR_INVALID_ARG, "cache_format %d invalid", c->cache_format);
  if (c->decay_mode != HLA_DECAY_SCALAR && c->decay_mode != HLA_DECAY_CHANNEL)
    return fail(HLA_ERR_INVALID_ARG, "decay_mode %d invalid", c->decay_mode);
  if (c->decay_mode == HLA_DECAY_CHANNEL && c->cache_format == HLA_CACHE_FACTORED)
    return fail(HLA_ERR_UNSUPPORTED, "a factored cache needs the scalar decay");
  if (c->pool_window != 0) {
    const int w = c->pool_window;
    if (w < 8 || w >= c->C || c->C % w != 0 || c->C / w > hla::kMaxWindows)
      return fail(HLA_ERR_UNSUPPORTED, "pool_window %d unsupported for C=%d (8 <= w < C, w | C, C / w <= %d)", w,
                  c->C, hla::kMaxWindows);
  }
  if (!(c->tau > 0.0f) || !std::isfinite(c->tau)) return fail(HLA_ERR_INVALID_ARG, "tau must be finite and > 0");
  if (!std::isfinite(c->bias) || !std::isfinite(c->skip_threshold))
    return fail(HLA_ERR_INVALID_ARG, "bias and skip_threshold must be finite");
  const double elems = (double)c->B * (need_T ? c->T : 1) * c->H * c->dk;
  if (elems > 9.0e15) return fail(HLA_ERR_UNSUPPORTED, "problem too large");
  return HLA_OK;
}

hla_status need_ptr(const void* p, const char* name) {
  if (p == nullptr) return fail(HLA_ERR_INVALID_ARG, "%s is NULL", name);
  if (!aligned16(p)) return fail(HLA_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
  return HLA_OK;
}

hla_status opt_ptr(const void* p, const char* name) {
  if (p != nullptr && !aligned16(p)) return fail(HLA_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
  return HLA_OK;
}

#define HLA_TRY(expr)                \
  do {                               \
    hla_status _s = (expr);          \
    if (_s != HLA_OK) return _s;     \
  } while (0)

#define HLA_CUDA(expr, where)                   \
  do {                                          \
    cudaError_t _e = (expr);                    \
    if (_e != cudaSuccess) return cuda_fail(_e, where); \
  } while (0)

float gate_scale(int d) { return (float)(1.0 / std::sqrt((double)d)); }

// Channel-wise decay (alpha with a trailing d_k axis).
bool chan(const hla_config* c) { return c->decay_mode == HLA_DECAY_CHANNEL; }

// Strides of the token-major alpha/beta view of [B,T,H] (scalar) or [B,T,H,d]
// (channel-wise decay: alpha strides are beta's times d).
void set_decay_view(hla::TokenView& in, const hla_config* c) {
  in.ab = (long)c->T * c->H;
  in.ah = 1;
  in.at = c->H;
  if (chan(c)) {
    in.ab *= c->dk;
    in.ah *= c->dk;
    in.at *= c->dk;
    in.alpha_vec = 1;
  }
}

// Window representatives per chunk (0: one pool per chunk) and key pools per chunk.
int n_windows(const hla_config* c) { return c->pool_window > 0 ? c->C / c->pool_window : 0; }
size_t key_reps(const hla_config* c) { return c->pool_window > 0 ? (size_t)(c->C / c->pool_window) : 1; }

// The WY solve and the intra-chunk read-out work on sub-chunks of kSub tokens; a
// chunk of C tokens is C / kSub of them.
constexpr int kSub = 64;

// Prefill workspace layout.
struct PrefillWs {
  size_t rq, rk, act_idx, act_g, act_cnt, order, A, Bm, Asub, Bsub, Wb, Ub, ell, S_in;
  size_t Kt, Kh, Kc, Qt, gC;  // channel-wise decay on the tensor cores: prepared operands
  size_t total;
};

// Channel-wise decay runs on the tensor cores for bf16 with d = 128 (the decays folded
// into the keys and queries per 64-token sub-chunk), else by the token rule on CUDA
// cores.
bool chan_tc(const hla_config* c) { return chan(c) && c->dtype == HLA_BF16 && c->dk == 128; }

PrefillWs prefill_layout(const hla_config* c) {
  PrefillWs w{};
  const size_t B = c->B, H = c->H, d = c->dk, C = c->C;
  const size_t N = (c->T + C - 1) / C;
  const size_t Nc = c->T / C;
  const size_t Nsub = (c->T + kSub - 1) / kSub;
  const size_t Nsub_c = c->T / kSub;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  w.rq = take(B * H * N * d * 4);
  w.rk = take(B * H * N * key_reps(c) * d * 4);
  w.act_idx = take(B * H * N * N * 4);
  w.act_g = take(B * H * N * N * 4);
  w.act_cnt = take(B * H * N * 4);
  w.order = take(B * H * N * 4);
  w.A = take(B * H * Nc * d * d * esize(c->dtype));
  w.Bm = take(B * H * Nc * d * d * esize(c->dtype));
  if (chan(c) && !chan_tc(c)) {  // token-rule transitions and read-out per chunk: no WY factors
    w.S_in = take(B * H * N * d * d * 4);
    w.total = off;
    return w;
  }
  if (chan_tc(c)) {  // Kt, Kh, Kc, Qt [B,H,Nsub,64,d] bf16 and gamma_C [B,H,Nsub,d] float32
    w.Kt = take(B * H * Nsub * kSub * d * 2);
    w.Kh = take(B * H * Nsub * kSub * d * 2);
    w.Kc = take(B * H * Nsub * kSub * d * 2);
    w.Qt = take(B * H * Nsub * kSub * d * 2);
    w.gC = take(B * H * Nsub * d * 4);
  }
  if (C > kSub) {  // transitions of the complete sub-chunks, merged into A, Bm
    w.Asub = take(B * H * Nsub_c * d * d * esize(c->dtype));
    w.Bsub = take(B * H * Nsub_c * d * d * esize(c->dtype));
  }
  w.Wb = take(B * H * Nsub * kSub * d * 4);
  w.Ub = take(B * H * Nsub * kSub * d * 4);
  w.ell = take(B * H * Nsub * kSub * 4);
  w.S_in = take(B * H * Nsub * d * d * 4);  // the state entering every sub-chunk
  w.total = off;
  return w;
}

struct CacheLayout {
  size_t A, Bm, Kf, Wf, Uf, df, rk, bk, bv, bqr, bkr, balpha, bbeta, n, m, total;
};

// Scales stored per chunk in a factored cache: gamma_C / gamma_t for t < C, then
// gamma_C, padded to a 16-byte multiple.
inline size_t df_stride(size_t C) { return C + 4; }

CacheLayout cache_layout(const hla_config* c, int32_t maxc) {
  CacheLayout L{};
  const size_t B = c->B, H = c->H, d = c->dk, C = c->C, es = esize(c->dtype);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  if (c->cache_format == HLA_CACHE_FACTORED) {
    L.Kf = take(B * H * (size_t)maxc * C * d * es);
    L.Wf = take(B * H * (size_t)maxc * C * d * es);
    L.Uf = take(B * H * (size_t)maxc * C * d * es);
    L.df = take(B * H * (size_t)maxc * df_stride(C) * 4);
  } else {
    L.A = take(B * H * (size_t)maxc * d * d * es);
    L.Bm = take(B * H * (size_t)maxc * d * d * es);
  }
  L.rk = take(B * H * (size_t)maxc * key_reps(c) * d * 4);
  L.bk = take(B * H * C * d * es);
  L.bv = take(B * H * C * d * es);
  L.bqr = take(B * H * C * d * es);
  L.bkr = take(B * H * C * d * es);
  L.balpha = take(B * H * C * (chan(c) ? d : 1) * 4);
  L.bbeta = take(B * H * C * 4);
  L.n = take(B * 4);
  L.m = take(B * 4);
  L.total = off;
  return L;
}

hla_status check_cache(const hla_config* c, const hla_cache* k) {
  if (k == nullptr) return fail(HLA_ERR_INVALID_ARG, "cache is NULL");
  if (k->B != c->B || k->H != c->H || k->C != c->C || k->d != c->dk || k->dtype != c->dtype ||
      k->format != c->cache_format || k->pool_window != c->pool_window || k->decay_mode != c->decay_mode)
    return fail(HLA_ERR_INVALID_ARG, "cache was initialised for a different config");
  if (k->max_chunks <= 0) return fail(HLA_ERR_INVALID_ARG, "cache max_chunks must be positive");
  const void* ps[] = {k->rk, k->buf_k, k->buf_v, k->buf_qr, k->buf_kr, k->buf_alpha, k->buf_beta};
  for (const void* p : ps) HLA_TRY(need_ptr(p, "cache buffer"));
  if (k->format == HLA_CACHE_FACTORED) {
    const void* fs[] = {k->Kf, k->Wf, k->Uf, k->df};
    for (const void* p : fs) HLA_TRY(need_ptr(p, "cache factor buffer"));
  } else {
    HLA_TRY(need_ptr(k->A, "cache A"));
    HLA_TRY(need_ptr(k->Bm, "cache B"));
  }
  // the per-sequence counters are read and written as single int32 values, so a
  // slice starting at any sequence is valid
  for (const int32_t* p : {k->n_chunks, k->m_partial})
    if (p == nullptr || ((uintptr_t)p & 3u) != 0) return fail(HLA_ERR_INVALID_ARG, "cache counters NULL or misaligned");
  return HLA_OK;
}

// ---- stage timing ------------------------------------------------------------
struct StagePair {
  cudaEvent_t a, b;
  int stage;
};
std::mutex g_prof_mu;
bool g_prof_on = false;
std::vector<StagePair> g_prof_pending;
double g_prof_ms[HLA_STAGE_COUNT] = {};
long g_prof_launches[HLA_STAGE_COUNT] = {};

// Records events around one stage on `stream` while profiling is on.
class StageScope {
 public:
  StageScope(int stage, cudaStream_t s, int launches) : stage_(stage), s_(s) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    if (!g_prof_on) return;
    if (cudaEventCreate(&a_) != cudaSuccess || cudaEventCreate(&b_) != cudaSuccess) return;
    cudaEventRecord(a_, s_);
    g_prof_launches[stage] += launches;
    on_ = true;
  }
  ~StageScope() {
    if (!on_) return;
    cudaEventRecord(b_, s_);
    std::lock_guard<std::mutex> lk(g_prof_mu);
    g_prof_pending.push_back({a_, b_, stage_});
  }

 private:
  int stage_;
  cudaStream_t s_;
  cudaEvent_t a_ = nullptr, b_ = nullptr;
  bool on_ = false;
};

// ---- CUDA context identity ----------------------------------------------------------
// Streams, events and symbol addresses belong to the CUDA context that was current
// when they were made.  The library keeps such handles per device and remembers the
// unique id of the context they belong to; a call made under another context (a
// non-primary one, or the primary context recreated after cudaDeviceReset) makes
// new ones.  The id comes from the driver API through the runtime's entry-point
// query, so the library does not link against the driver library.
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Id of the context current on this thread; 0 if none is current or the driver
// does not provide the calls.
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = (CtxGetCurrentFn)p;
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = (CtxGetIdFn)p;
  });
  if (get_current == nullptr || get_id == nullptr) return 0;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  unsigned long long id = 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// ---- side stream ---------------------------------------------------------------
// hla_prefill runs the routing stage (pools, gates, active lists) on a per-device
// side stream, forked from and joined back to the caller's stream by events, so it
// overlaps the chunk transitions: the two read only the caller's inputs and write
// disjoint parts of the workspace.  Created on first use on each device (and again
// when the current context is not the one it was made in).  One lock covers every
// device's side stream: concurrent hla_prefill calls, on any streams, enqueue their
// routing one after another through it.
struct SideStream {
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
  unsigned long long ctx_id = 0;
};
constexpr int kMaxDevices = 64;
std::mutex g_side_mu;
SideStream g_side[kMaxDevices];

// Makes `s` wait for the routing enqueued on the side stream.  Armed once the
// side stream has forked from `s`; an error return before the regular join runs
// it, so the caller's stream (or a capture on it) never holds an unjoined fork.
struct SideJoin {
  cudaStream_t side = nullptr, s = nullptr;
  cudaEvent_t join = nullptr;
  bool armed = false;
  ~SideJoin() {
    if (!armed) return;
    cudaEventRecord(join, side);
    cudaStreamWaitEvent(s, join, 0);
  }
};

hla_status side_stream(SideStream** out) {
  int dev = -1;
  HLA_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(HLA_ERR_UNSUPPORTED, "device ordinal %d beyond %d", dev, kMaxDevices);
  SideStream& ss = g_side[dev];
  // handles of another context are dropped, not destroyed (that context may be gone)
  if (ss.s != nullptr && ss.ctx_id != current_context_id()) ss = SideStream{};
  if (ss.s == nullptr) {
    cudaStream_t st = nullptr;
    cudaEvent_t f = nullptr, j = nullptr;
    HLA_CUDA(cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking), "side stream create");
    HLA_CUDA(cudaEventCreateWithFlags(&f, cudaEventDisableTiming), "side stream event create");
    HLA_CUDA(cudaEventCreateWithFlags(&j, cudaEventDisableTiming), "side stream event create");
    ss.fork = f;
    ss.join = j;
    ss.s = st;
    ss.ctx_id = current_context_id();
  }
  *out = &ss;
  return HLA_OK;
}

}  // namespace

extern "C" {

const char* hla_last_error(void) { return g_msg; }

size_t hla_cache_bytes(const hla_config* cfg, int32_t max_chunks) {
  if (check_cfg(cfg, false) != HLA_OK || max_chunks <= 0) return 0;
  return cache_layout(cfg, max_chunks).total;
}

hla_status hla_cache_init(const hla_config* cfg, int32_t max_chunks, void* mem, size_t bytes, hla_cache* out,
                          hla_stream_t stream) {
  g_msg[0] = 0;
  HLA_TRY(check_cfg(cfg, false));
  if (out == nullptr) return fail(HLA_ERR_INVALID_ARG, "out is NULL");
  if (max_chunks <= 0) return fail(HLA_ERR_INVALID_ARG, "max_chunks must be positive");
  HLA_TRY(need_ptr(mem, "mem"));
  if (((uintptr_t)mem & 255u) != 0) return fail(HLA_ERR_INVALID_ARG, "cache memory must be 256-byte aligned");
  if (cfg->cache_format == HLA_CACHE_FACTORED && !(cfg->dtype == HLA_BF16 && cfg->dk == 128 && cfg->C == 64))
    return fail(HLA_ERR_UNSUPPORTED, "a factored cache needs bf16, d = 128 and C = 64");
  if (cfg->cache_format == HLA_CACHE_FACTORED && chan(cfg))
    return fail(HLA_ERR_UNSUPPORTED, "a factored cache needs the scalar decay");
  const CacheLayout L = cache_layout(cfg, max_chunks);
  if (bytes < L.total) return fail(HLA_ERR_WORKSPACE, "cache block too small: %zu < %zu", bytes, L.total);
  char* base = (char*)mem;
  hla_cache c{};
  c.max_chunks = max_chunks;
  c.B = cfg->B;
  c.H = cfg->H;
  c.C = cfg->C;
  c.d = cfg->dk;
  c.dtype = cfg->dtype;
  c.format = cfg->cache_format;
  c.pool_window = cfg->pool_window;
  c.decay_mode = cfg->decay_mode;
  if (cfg->cache_format == HLA_CACHE_FACTORED) {
    c.Kf = base + L.Kf;
    c.Wf = base + L.Wf;
    c.Uf = base + L.Uf;
    c.df = (float*)(base + L.df);
  } else {
    c.A = base + L.A;
    c.Bm = base + L.Bm;
  }
  c.rk = (float*)(base + L.rk);
  c.buf_k = base + L.bk;
  c.buf_v = base + L.bv;
  c.buf_qr = base + L.bqr;
  c.buf_kr = base + L.bkr;
  c.buf_alpha = (float*)(base + L.balpha);
  c.buf_beta = (float*)(base + L.bbeta);
  c.n_chunks = (int32_t*)(base + L.n);
  c.m_partial = (int32_t*)(base + L.m);
  HLA_CUDA(cudaMemsetAsync(base + L.n, 0, L.total - L.n, (cudaStream_t)stream), "hla_cache_init memset");
  *out = c;
  return HLA_OK;
}

hla_status hla_cache_slice(const hla_cache* cache, int32_t b0, int32_t nb, hla_cache* out) {
  g_msg[0] = 0;
  if (cache == nullptr || out == nullptr) return fail(HLA_ERR_INVALID_ARG, "cache and out must not be NULL");
  if (cache->B <= 0 || cache->H <= 0 || cache->max_chunks <= 0 || cache->d <= 0 || cache->C <= 0)
    return fail(HLA_ERR_INVALID_ARG, "cache is not initialised");
  if (b0 < 0 || nb < 1 || (int64_t)b0 + nb > cache->B)
    return fail(HLA_ERR_INVALID_ARG, "sequences [%d, %d) outside the cache's %d", b0, b0 + nb, cache->B);
  // per-sequence bytes of each buffer (the layout of cache_layout, sequence-major)
  const size_t H = cache->H, d = cache->d, C = cache->C, mc = cache->max_chunks;
  const size_t es = esize(cache->dtype);
  const size_t off = (size_t)b0;
  hla_cache v = *cache;
  v.B = nb;
  if (cache->format == HLA_CACHE_FACTORED) {
    v.Kf = (char*)cache->Kf + off * H * mc * C * d * es;
    v.Wf = (char*)cache->Wf + off * H * mc * C * d * es;
    v.Uf = (char*)cache->Uf + off * H * mc * C * d * es;
    v.df = (float*)((char*)cache->df + off * H * mc * df_stride(C) * 4);
  } else {
    v.A = (char*)cache->A + off * H * mc * d * d * es;
    v.Bm = (char*)cache->Bm + off * H * mc * d * d * es;
  }
  const size_t reps = cache->pool_window > 0 ? (size_t)(cache->C / cache->pool_window) : 1;
  v.rk = (float*)((char*)cache->rk + off * H * mc * reps * d * 4);
  v.buf_k = (char*)cache->buf_k + off * H * C * d * es;
  v.buf_v = (char*)cache->buf_v + off * H * C * d * es;
  v.buf_qr = (char*)cache->buf_qr + off * H * C * d * es;
  v.buf_kr = (char*)cache->buf_kr + off * H * C * d * es;
  const size_t adim = cache->decay_mode == HLA_DECAY_CHANNEL ? d : 1;
  v.buf_alpha = (float*)((char*)cache->buf_alpha + off * H * C * adim * 4);
  v.buf_beta = (float*)((char*)cache->buf_beta + off * H * C * 4);
  v.n_chunks = cache->n_chunks + off;
  v.m_partial = cache->m_partial + off;
  *out = v;
  return HLA_OK;
}

size_t hla_prefill_workspace_bytes(const hla_config* cfg) {
  if (check_cfg(cfg, true) != HLA_OK) return 0;
  return prefill_layout(cfg).total;
}

size_t hla_decode_workspace_bytes(const hla_config* cfg, int32_t max_chunks) {
  if (check_cfg(cfg, false) != HLA_OK || max_chunks <= 0) return 0;
  const size_t n = (size_t)cfg->B * cfg->H * max_chunks;
  // active lists and gates [B,H,max_chunks], then one list length per (sequence, head)
  return align256(n * 4) + align256(n * 4) + align256((size_t)cfg->B * cfg->H * 4);
}

hla_status gdn_chunk_transitions(const hla_config* cfg, const void* k, const void* v, const float* alpha,
                                 const float* beta, void* A_out, void* B_out, hla_stream_t stream) {
  g_msg[0] = 0;
  HLA_TRY(check_cfg(cfg, true));
  HLA_TRY(need_ptr(k, "k"));
  HLA_TRY(need_ptr(v, "v"));
  HLA_TRY(need_ptr(alpha, "alpha"));
  HLA_TRY(need_ptr(beta, "beta"));
  HLA_TRY(need_ptr(A_out, "A_out"));
  HLA_TRY(need_ptr(B_out, "B_out"));
  const int Nc = cfg->T / cfg->C;
  if (Nc == 0) return HLA_OK;
  hla::TransArgs t{};
  t.B = cfg->B;
  t.H = cfg->H;
  t.T = Nc * cfg->C;
  t.C = cfg->C;
  t.d = cfg->dk;
  t.dtype = cfg->dtype;
  t.in = {k, v, alpha, beta, (long)cfg->T * cfg->H * cfg->dk, cfg->dk, (long)cfg->H * cfg->dk,
          (long)cfg->T * cfg->H, 1, cfg->H};
  set_decay_view(t.in, cfg);
  t.n_chunks = Nc;
  t.A = A_out;
  t.Bm = B_out;
  t.ab_chunk_stride = Nc;
  // channel-wise decay, or no workspace here for sub-chunk factors: the token rule
  if (cfg->C > kSub || chan(cfg))
    HLA_CUDA(hla::launch_transitions_token(t, (cudaStream_t)stream), "gdn_chunk_transitions (token rule) launch");
  else if (cfg->dtype == HLA_BF16 && cfg->dk == 128)
    HLA_CUDA(hla::launch_transitions_tc(t, (cudaStream_t)stream), "gdn_chunk_transitions (tensor core) launch");
  else
    HLA_CUDA(hla::launch_transitions(t, (cudaStream_t)stream), "gdn_chunk_transitions launch");
  return HLA_OK;
}

// Query pools per chunk and key pools per chunk, or per window with window
// representatives (window u of chunk j at row j * W + u).
static hla_status launch_route_pools(const hla_config* cfg, const void* q_route, const void* k_route, float* rq,
                                     float* rk, cudaStream_t s) {
  const int N = (cfg->T + cfg->C - 1) / cfg->C;
  if (cfg->pool_window == 0) {
    HLA_CUDA(hla::launch_pools(q_route, k_route, rq, rk, cfg->B, cfg->T, cfg->H, cfg->dk, cfg->C, N, cfg->tau,
                               cfg->dtype, s),
             "pool launch");
    return HLA_OK;
  }
  if (q_route != nullptr && rq != nullptr)
    HLA_CUDA(hla::launch_pools(q_route, nullptr, rq, nullptr, cfg->B, cfg->T, cfg->H, cfg->dk, cfg->C, N, cfg->tau,
                               cfg->dtype, s),
             "query pool launch");
  if (k_route != nullptr && rk != nullptr)
    HLA_CUDA(hla::launch_pools(nullptr, k_route, nullptr, rk, cfg->B, cfg->T, cfg->H, cfg->dk, cfg->pool_window,
                               N * n_windows(cfg), cfg->tau, cfg->dtype, s),
             "window pool launch");
  return HLA_OK;
}

static hla_status routing_impl(const hla_config* cfg, const void* q_route, const void* k_route, float* rq,
                               float* rk, const float* user_gates, int32_t* act_idx, float* act_g,
                               int32_t* act_cnt, float* gates_out, int32_t* active_idx_out,
                               int32_t* active_cnt_out, cudaStream_t s) {
  const int N = (cfg->T + cfg->C - 1) / cfg->C;
  if (cfg->gate_mode == HLA_GATES_ROUTED || rk != nullptr) {
    const bool routed = cfg->gate_mode == HLA_GATES_ROUTED;
    StageScope _sc(HLA_STAGE_POOLS, s, cfg->pool_window > 0 ? 2 : 1);
    HLA_TRY(launch_route_pools(cfg, routed ? q_route : nullptr, k_route, routed ? rq : nullptr, rk, s));
  }
  hla::GatesArgs g{};
  g.B = cfg->B;
  g.H = cfg->H;
  g.N = N;
  g.d = cfg->dk;
  g.mode = cfg->gate_mode;
  g.win = n_windows(cfg);
  g.c_d = gate_scale(cfg->dk);
  g.bias = cfg->bias;
  g.thr = cfg->skip_threshold;
  g.rq = rq;
  g.rk = rk;
  g.user_gates = user_gates;
  g.act_idx = act_idx;
  g.act_g = act_g;
  g.act_cnt = act_cnt;
  g.gates_out = gates_out;
  g.active_idx_out = active_idx_out;
  g.active_cnt_out = active_cnt_out;
  {
    StageScope _sc(HLA_STAGE_GATES, s, 1);
    HLA_CUDA(hla::launch_gates(g, s), "gates launch");
  }
  return HLA_OK;
}

hla_status hla_routing(const hla_config* cfg, const void* q_route, const void* k_route, float* rq_out,
                       float* rk_out, float* gates_out, int32_t* active_idx_out, int32_t* active_cnt_out,
                       hla_stream_t stream) {
  g_msg[0] = 0;
  HLA_TRY(check_cfg(cfg, true));
  if (cfg->gate_mode == HLA_GATES_USER) return fail(HLA_ERR_UNSUPPORTED, "hla_routing does not take user gates");
  HLA_TRY(need_ptr(q_route, "q_route"));
  HLA_TRY(need_ptr(k_route, "k_route"));
  HLA_TRY(need_ptr(rq_out, "rq_out"));
  HLA_TRY(need_ptr(rk_out, "rk_out"));
  HLA_TRY(opt_ptr(gates_out, "gates_out"));
  HLA_TRY(opt_ptr(active_idx_out, "active_idx_out"));
  HLA_TRY(opt_ptr(active_cnt_out, "active_cnt_out"));
  if ((active_idx_out == nullptr) != (active_cnt_out == nullptr))
    return fail(HLA_ERR_INVALID_ARG, "active_idx_out and active_cnt_out go together");
  const int N = (cfg->T + cfg->C - 1) / cfg->C;
  cudaStream_t s = (cudaStream_t)stream;
  HLA_TRY(launch_route_pools(cfg, q_route, k_route, rq_out, rk_out, s));
  hla::GatesArgs g{};
  g.B = cfg->B;
  g.H = cfg->H;
  g.N = N;
  g.d = cfg->dk;
  g.mode = cfg->gate_mode;
  g.win = n_windows(cfg);
  g.c_d = gate_scale(cfg->dk);
  g.bias = cfg->bias;
  g.thr = cfg->skip_threshold;
  g.rq = rq_out;
  g.rk = rk_out;
  g.act_idx = active_idx_out;
  g.act_cnt = active_cnt_out;
  g.pad_act_idx = true;
  g.gates_out = gates_out;
  HLA_CUDA(hla::launch_gates(g, s), "gates launch");
  return HLA_OK;
}

hla_status hla_gate_support(const hla_config* cfg, const float* gates, float* mass_out, float* support_out,
                            hla_stream_t stream) {
  g_msg[0] = 0;
  HLA_TRY(check_cfg(cfg, true));
  HLA_TRY(need_ptr(gates, "gates"));
  HLA_TRY(opt_ptr(mass_out, "mass_out"));
  HLA_TRY(opt_ptr(support_out, "support_out"));
  if (mass_out == nullptr && support_out == nullptr)
    return fail(HLA_ERR_INVALID_ARG, "mass_out and support_out are both NULL");
  const int N = (cfg->T + cfg->C - 1) / cfg->C;
  if ((double)cfg->B * cfg->H * N >= 2147483647.0) return fail(HLA_ERR_UNSUPPORTED, "too many gate rows");
  HLA_CUDA(hla::launch_gate_support(gates, cfg->B, cfg->H, N, cfg->skip_threshold, mass_out, support_out,
                                    (cudaStream_t)stream),
           "gate support launch");
  return HLA_OK;
}

hla_status hla_prefill(const hla_config* cfg, const void* q, const void* k, const void* v, const float* alpha,
                       const float* beta, const void* q_route, const void* k_route, const float* user_gates,
                       void* o, float* gates_out, int32_t* active_idx_out, int32_t* active_cnt_out,
                       hla_cache* cache_out, void* workspace, size_t workspace_bytes, hla_stream_t stream) {
  g_msg[0] = 0;
  HLA_TRY(check_cfg(cfg, true));
  HLA_TRY(need_ptr(q, "q"));
  HLA_TRY(need_ptr(k, "k"));
  HLA_TRY(need_ptr(v, "v"));
  HLA_TRY(need_ptr(alpha, "alpha"));
  HLA_TRY(need_ptr(beta, "beta"));
  HLA_TRY(need_ptr(o, "o"));
  HLA_TRY(opt_ptr(q_route, "q_route"));
  HLA_TRY(opt_ptr(k_route, "k_route"));
  HLA_TRY(opt_ptr(gates_out, "gates_out"));
  HLA_TRY(opt_ptr(active_idx_out, "active_idx_out"));
  HLA_TRY(opt_ptr(active_cnt_out, "active_cnt_out"));
  if (cfg->gate_mode == HLA_GATES_USER) HLA_TRY(need_ptr(user_gates, "user_gates"));
  const int N = (cfg->T + cfg->C - 1) / cfg->C;
  const int Nc = cfg->T / cfg->C;
  if (cache_out != nullptr) {
    HLA_TRY(check_cache(cfg, cache_out));
    if (cache_out->max_chunks < Nc)
      return fail(HLA_ERR_WORKSPACE, "cache holds %d chunks, prompt has %d", cache_out->max_chunks, Nc);
  }
  const PrefillWs w = prefill_layout(cfg);
  HLA_TRY(need_ptr(workspace, "workspace"));
  if (((uintptr_t)workspace & 255u) != 0) return fail(HLA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (workspace_bytes < w.total)
    return fail(HLA_ERR_WORKSPACE, "workspace too small: %zu < %zu", workspace_bytes, w.total);
  char* ws = (char*)workspace;
  cudaStream_t s = (cudaStream_t)stream;
  // bf16 with d = 128 runs on the tensor cores (bf16 WY factors and S_in in the
  // workspace); other shapes run the float32 CUDA-core kernels.
  const bool tc_path = cfg->dtype == HLA_BF16 && cfg->dk == 128;
  const void* qr = q_route ? q_route : q;
  const void* kr = k_route ? k_route : k;
  float* rq = (float*)(ws + w.rq);
  float* rk = (float*)(ws + w.rk);
  int32_t* act_idx = (int32_t*)(ws + w.act_idx);
  float* act_g = (float*)(ws + w.act_g);
  int32_t* act_cnt = (int32_t*)(ws + w.act_cnt);
  // routing on the side stream, overlapping the transitions below; joined before the
  // composition (the fork/join pair is enqueued under one lock)
  std::unique_lock<std::mutex> side_lock(g_side_mu);
  SideStream* side = nullptr;
  HLA_TRY(side_stream(&side));
  HLA_CUDA(cudaEventRecord(side->fork, s), "side stream fork");
  HLA_CUDA(cudaStreamWaitEvent(side->s, side->fork, 0), "side stream fork");
  SideJoin side_join;
  side_join.side = side->s;
  side_join.s = s;
  side_join.join = side->join;
  side_join.armed = true;
  HLA_TRY(routing_impl(cfg, qr, kr, rq, (cfg->gate_mode == HLA_GATES_ROUTED || cache_out) ? rk : nullptr,
                       user_gates, act_idx, act_g, act_cnt, gates_out, active_idx_out, active_cnt_out, side->s));
  HLA_CUDA(cudaEventRecord(side->join, side->s), "side stream join");
  // transitions of every 64-token sub-chunk (A/B of complete ones into the cache or
  // workspace; at C > 64 into the workspace, merged per chunk below)
  // Channel-wise decay: the token rule over whole chunks, no sub-chunks (float32, or
  // d = 64); bf16 with d = 128 takes the tensor-core path below with the decays folded
  // into prepared keys and queries (chan_tc_path).
  const bool chan_path = chan(cfg) && !chan_tc(cfg);
  const bool chan_tc_path = chan_tc(cfg);
  const int s_sub = chan_path ? 1 : cfg->C / kSub;
  const int Nsub = chan_path ? N : (cfg->T + kSub - 1) / kSub;
  const int Nsub_c = chan_path ? Nc : cfg->T / kSub;
  hla::TransArgs t{};
  t.B = cfg->B;
  t.H = cfg->H;
  t.T = cfg->T;
  t.C = chan_path ? cfg->C : kSub;
  t.d = cfg->dk;
  t.dtype = cfg->dtype;
  t.in = {k, v, alpha, beta, (long)cfg->T * cfg->H * cfg->dk, cfg->dk, (long)cfg->H * cfg->dk,
          (long)cfg->T * cfg->H, 1, cfg->H};
  set_decay_view(t.in, cfg);
  t.n_chunks = Nsub;
  // a dense cache takes A/B straight from the transitions (or the merge); otherwise
  // they go to the workspace (the composition reads them) and a factored cache gets
  // the WY factors
  const bool dense_out = cache_out != nullptr && cache_out->format == HLA_CACHE_DENSE;
  void* A_chunk = dense_out ? cache_out->A : (void*)(ws + w.A);
  void* B_chunk = dense_out ? cache_out->Bm : (void*)(ws + w.Bm);
  const long chunk_stride = dense_out ? cache_out->max_chunks : Nc;
  if (s_sub == 1) {
    t.A = A_chunk;
    t.Bm = B_chunk;
    t.ab_chunk_stride = chunk_stride;
  } else {
    t.A = ws + w.Asub;
    t.Bm = ws + w.Bsub;
    t.ab_chunk_stride = Nsub_c;
  }
  t.Wb = chan_path ? nullptr : (float*)(ws + w.Wb);
  t.Ub = chan_path ? nullptr : (float*)(ws + w.Ub);
  t.ell = (chan_path || chan_tc_path) ? nullptr : (float*)(ws + w.ell);
  hla::ChanOperands ops{};
  if (chan_tc_path) {
    ops.Kt = ws + w.Kt;
    ops.Kh = ws + w.Kh;
    ops.Kc = ws + w.Kc;
    ops.Qt = ws + w.Qt;
    ops.gC = (const float*)(ws + w.gC);
  }
  {
    StageScope _sc(HLA_STAGE_TRANSITIONS, s, chan_tc_path ? 2 : 1);
    if (chan_tc_path) {
      hla::ChanPrepArgs pa{};
      pa.B = cfg->B;
      pa.H = cfg->H;
      pa.T = cfg->T;
      pa.Nsub = Nsub;
      pa.k = k;
      pa.q = q;
      pa.alpha = alpha;
      pa.Kt = ws + w.Kt;
      pa.Kh = ws + w.Kh;
      pa.Kc = ws + w.Kc;
      pa.Qt = ws + w.Qt;
      pa.gC = (float*)(ws + w.gC);
      HLA_CUDA(hla::launch_chan_prep(pa, s), "channel-decay operand launch");
      HLA_CUDA(hla::launch_transitions_tc(t, s, &ops), "transitions (tensor core, channel decay) launch");
    } else if (chan_path) {
      HLA_CUDA(hla::launch_transitions_token(t, s), "transitions (token rule) launch");
    } else if (tc_path) {
      HLA_CUDA(hla::launch_transitions_tc(t, s), "transitions (tensor core) launch");
    } else {
      HLA_CUDA(hla::launch_transitions(t, s), "transitions launch");
    }
  }
  // chunks of C > 64 tokens: each chunk's transition from its sub-chunks' ones
  hla::ChainArgs ch{};
  ch.B = cfg->B;
  ch.H = cfg->H;
  ch.d = cfg->dk;
  ch.dtype = cfg->dtype;
  ch.s = s_sub;
  ch.Asub = t.A;
  ch.Bsub = t.Bm;
  ch.sub_stride = Nsub_c;
  ch.Nc = Nc;
  ch.Aout = A_chunk;
  ch.Bout = B_chunk;
  ch.out_stride = chunk_stride;
  ch.N = N;
  ch.Nsub = Nsub;
  ch.S = ws + w.S_in;
  if (s_sub > 1 && Nc > 0) {
    StageScope _sc(HLA_STAGE_CHAIN, s, 1);
    HLA_CUDA(hla::launch_chain_merge(ch, s), "chunk merge launch");
  }
  side_join.armed = false;
  HLA_CUDA(cudaStreamWaitEvent(s, side->join, 0), "side stream join");
  side_lock.unlock();
  hla::ComposeArgs c{};
  c.B = cfg->B;
  c.H = cfg->H;
  c.N = N;
  c.d = cfg->dk;
  c.dtype = cfg->dtype;
  c.A = A_chunk;
  c.Bm = B_chunk;
  c.ab_chunk_stride = Nc > 0 ? chunk_stride : 0;
  c.act_idx = act_idx;
  c.act_g = act_g;
  c.act_cnt = act_cnt;
  c.S_in = (float*)(ws + w.S_in);
  c.slot_mult = s_sub;
  c.n_slots = Nsub;
  c.sparse = cfg->skip_threshold > 0.0f;
  c.order = (int32_t*)(ws + w.order);
  {
    StageScope _sc(HLA_STAGE_COMPOSE, s, 1);
    // every gate one (and kept): the composition is a plain prefix scan over the chunks
    const bool scan = cfg->gate_mode == HLA_GATES_ONE && cfg->skip_threshold <= 1.0f;
    if (tc_path)
      HLA_CUDA(hla::launch_compose_tc(c, scan, s), "compose (tensor core) launch");
    else
      HLA_CUDA(hla::launch_compose(c, s), "compose launch");
  }
  if (s_sub > 1 && Nsub > 1) {  // the state entering every later sub-chunk of each chunk
    StageScope _sc(HLA_STAGE_CHAIN, s, 1);
    HLA_CUDA(hla::launch_chain_advance(ch, s), "sub-chunk advance launch");
  }
  if (chan_path) {
    hla::ReadoutTokenArgs rt{};
    rt.B = cfg->B;
    rt.H = cfg->H;
    rt.T = cfg->T;
    rt.C = cfg->C;
    rt.N = N;
    rt.d = cfg->dk;
    rt.dtype = cfg->dtype;
    rt.in = t.in;
    rt.q = q;
    rt.S_in = c.S_in;
    rt.S_bf16 = tc_path;  // the tensor-core composition writes bf16 states
    rt.o = o;
    StageScope _sc(HLA_STAGE_READOUT, s, 1);
    HLA_CUDA(hla::launch_readout_token(rt, s), "readout (token rule) launch");
  }
  hla::ReadoutArgs r{};
  r.B = cfg->B;
  r.H = cfg->H;
  r.T = cfg->T;
  r.C = kSub;
  r.N = Nsub;
  r.d = cfg->dk;
  r.dtype = cfg->dtype;
  r.q = q;
  r.k = k;
  r.S_in = c.S_in;
  r.Wb = t.Wb;
  r.Ub = t.Ub;
  r.ell = t.ell;
  r.o = o;
  if (!chan_path) {
    StageScope _sc(HLA_STAGE_READOUT, s, 1);
    if (tc_path)
      HLA_CUDA(hla::launch_readout_tc(r, c.S_in, t.Wb, t.Ub, s, chan_tc_path ? &ops : nullptr),
               "readout (tensor core) launch");
    else
      HLA_CUDA(hla::launch_readout(r, s), "readout launch");
  }
  if (cache_out) {
    hla::DecodeArgs dc{};
    dc.B = cfg->B;
    dc.H = cfg->H;
    dc.C = cfg->C;
    dc.d = cfg->dk;
    dc.dtype = cfg->dtype;
    dc.max_chunks = cache_out->max_chunks;
    dc.win = n_windows(cfg);
    dc.alpha_vec = chan(cfg) ? 1 : 0;
    dc.rk = cache_out->rk;
    dc.buf_k = cache_out->buf_k;
    dc.buf_v = cache_out->buf_v;
    dc.buf_qr = cache_out->buf_qr;
    dc.buf_kr = cache_out->buf_kr;
    dc.buf_alpha = cache_out->buf_alpha;
    dc.buf_beta = cache_out->buf_beta;
    dc.n_chunks = cache_out->n_chunks;
    dc.m_partial = cache_out->m_partial;
    const bool factored = cache_out->format == HLA_CACHE_FACTORED;
    StageScope _sc(HLA_STAGE_CACHE, s, factored ? 2 : 1);
    HLA_CUDA(hla::launch_cache_fill(dc, rk, qr, kr, k, v, alpha, beta, cfg->T, s), "cache fill launch");
    if (factored && Nc > 0) {
      hla::FactorFillArgs f{};
      f.B = cfg->B;
      f.H = cfg->H;
      f.T = cfg->T;
      f.N = N;
      f.Nc = Nc;
      f.max_chunks = cache_out->max_chunks;
      f.k = k;
      f.Wb = ws + w.Wb;
      f.Ub = ws + w.Ub;
      f.ell = (const float*)(ws + w.ell);
      f.Kf = cache_out->Kf;
      f.Wf = cache_out->Wf;
      f.Uf = cache_out->Uf;
      f.df = cache_out->df;
      HLA_CUDA(hla::launch_factor_fill(f, s), "factor fill launch");
    }
  }
  return HLA_OK;
}

hla_status hla_decode_step(const hla_config* cfg, hla_cache* cache, const void* q, const void* k, const void* v,
                           const float* alpha, const float* beta, const void* q_route, const void* k_route,
                           void* o, void* workspace, size_t workspace_bytes, hla_stream_t stream) {
  g_msg[0] = 0;
  HLA_TRY(check_cfg(cfg, false));
  if (cfg->gate_mode == HLA_GATES_USER) return fail(HLA_ERR_UNSUPPORTED, "decode does not take user gates");
  HLA_TRY(check_cache(cfg, cache));
  HLA_TRY(need_ptr(q, "q"));
  HLA_TRY(need_ptr(k, "k"));
  HLA_TRY(need_ptr(v, "v"));
  HLA_TRY(need_ptr(alpha, "alpha"));
  HLA_TRY(need_ptr(beta, "beta"));
  HLA_TRY(need_ptr(o, "o"));
  HLA_TRY(opt_ptr(q_route, "q_route"));
  HLA_TRY(opt_ptr(k_route, "k_route"));
  const size_t need = hla_decode_workspace_bytes(cfg, cache->max_chunks);
  HLA_TRY(need_ptr(workspace, "workspace"));
  if (((uintptr_t)workspace & 255u) != 0) return fail(HLA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (workspace_bytes < need) return fail(HLA_ERR_WORKSPACE, "workspace too small: %zu < %zu", workspace_bytes, need);
  hla::DecodeArgs a{};
  a.B = cfg->B;
  a.H = cfg->H;
  a.C = cfg->C;
  a.d = cfg->dk;
  a.dtype = cfg->dtype;
  a.mode = cfg->gate_mode;
  a.max_chunks = cache->max_chunks;
  a.win = n_windows(cfg);
  a.alpha_vec = chan(cfg) ? 1 : 0;
  a.tau = cfg->tau;
  a.c_d = gate_scale(cfg->dk);
  a.bias = cfg->bias;
  a.thr = cfg->skip_threshold;
  a.q = q;
  a.k = k;
  a.v = v;
  a.alpha = alpha;
  a.beta = beta;
  a.q_route = q_route;
  a.k_route = k_route;
  a.o = o;
  a.A = cache->A;
  a.Bm = cache->Bm;
  a.format = cache->format;
  a.Kf = cache->Kf;
  a.Wf = cache->Wf;
  a.Uf = cache->Uf;
  a.df = cache->df;
  a.rk = cache->rk;
  a.buf_k = cache->buf_k;
  a.buf_v = cache->buf_v;
  a.buf_qr = cache->buf_qr;
  a.buf_kr = cache->buf_kr;
  a.buf_alpha = cache->buf_alpha;
  a.buf_beta = cache->buf_beta;
  a.n_chunks = cache->n_chunks;
  a.m_partial = cache->m_partial;
  const size_t n = (size_t)cfg->B * cfg->H * cache->max_chunks;
  a.act_idx = (int32_t*)workspace;
  a.act_g = (float*)((char*)workspace + align256(n * 4));
  a.act_cnt = (int32_t*)((char*)workspace + 2 * align256(n * 4));
  cudaStream_t s = (cudaStream_t)stream;
  {
    // the dense bf16 cache with d = 128 gates in one kernel and streams in another
    const bool two = cache->format == HLA_CACHE_DENSE && cfg->dtype == HLA_BF16 && cfg->dk == 128;
    StageScope _sc(HLA_STAGE_DECODE, s, two ? 2 : 1);
    HLA_CUDA(hla::launch_decode_main(a, s), "decode launch");
  }
  {
    StageScope _sc(HLA_STAGE_DECODE_CLOSE, s, 3);
    HLA_CUDA(hla::launch_decode_close(a, s), "decode close launch");
  }
  return HLA_OK;
}

// ---------------------------------------------------------------------------
// Decode step with library-owned scratch.
//
// hla_decode_step wants the caller to hand it a device scratch block (the
// per-head list of active chunks and their gates).  A caller that may not
// allocate device memory at the point where it decodes -- a plug-in inside a
// runtime that owns every byte through its own pool and forbids allocations by
// its extensions, or a host thread that runs decode without an allocator in
// reach -- uses hla_decode_step_static instead.  Its scratch is the fixed array
// below: statically sized device memory of this library, looked up once per
// device, never allocated or freed by any call.
//
// Every call on a device uses the same array.  Nothing in it must start at
// zero (each decode kernel writes every entry it later reads), but two calls
// whose kernels overlap in time -- on different streams, or from different
// host threads -- write the same bytes and race: the caller serialises them.
// ---------------------------------------------------------------------------
namespace {
constexpr size_t kStaticScratchBytes = HLA_DECODE_STATIC_SCRATCH_BYTES;
constexpr int kStaticMaxDevices = 64;
std::mutex g_static_mu;
void* g_static_ptr[kStaticMaxDevices] = {};
unsigned long long g_static_ctx[kStaticMaxDevices] = {};
}  // namespace

static __device__ __align__(256) unsigned char hla_static_scratch[kStaticScratchBytes];

namespace {
// Device address of hla_static_scratch on the current device.  The first call on
// a device asks the runtime for the symbol's address (with that device current);
// later calls reuse it while the same CUDA context is current.  A different
// context -- a non-primary one, or the primary context recreated after
// cudaDeviceReset -- has its own copy of the array, so the address is looked up
// again.
hla_status static_scratch_ptr(void** out) {
  int dev = -1;
  HLA_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  if (dev < 0 || dev >= kStaticMaxDevices)
    return fail(HLA_ERR_UNSUPPORTED, "device ordinal %d beyond %d", dev, kStaticMaxDevices);
  std::lock_guard<std::mutex> lk(g_static_mu);
  const unsigned long long ctx = current_context_id();
  if (g_static_ptr[dev] == nullptr || ctx == 0 || ctx != g_static_ctx[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, hla_static_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(hla_static_scratch)");
    if (p == nullptr || ((uintptr_t)p & 255u) != 0)
      return fail(HLA_ERR_CUDA, "static scratch address %p is not 256-byte aligned", p);
    g_static_ptr[dev] = p;
    g_static_ctx[dev] = current_context_id();  // the lookup makes the context current if none was
  }
  *out = g_static_ptr[dev];
  return HLA_OK;
}
}  // namespace

hla_status hla_decode_step_static(const hla_config* cfg, hla_cache* cache, const void* q, const void* k,
                                  const void* v, const float* alpha, const float* beta, const void* q_route,
                                  const void* k_route, void* o, hla_stream_t stream) {
  g_msg[0] = 0;
  HLA_TRY(check_cfg(cfg, false));
  HLA_TRY(check_cache(cfg, cache));
  const size_t need = hla_decode_workspace_bytes(cfg, cache->max_chunks);
  if (need > kStaticScratchBytes)
    return fail(HLA_ERR_WORKSPACE,
                "decode scratch for B=%d H=%d max_chunks=%d is %zu bytes; the static array holds %zu "
                "(8 B per (sequence, head, chunk) and 4 B per (sequence, head), each part rounded up to "
                "256 B); use hla_decode_step with a caller workspace",
                cfg->B, cfg->H, cache->max_chunks, need, kStaticScratchBytes);
  void* ws = nullptr;
  HLA_TRY(static_scratch_ptr(&ws));
  return hla_decode_step(cfg, cache, q, k, v, alpha, beta, q_route, k_route, o, ws, kStaticScratchBytes, stream);
}

hla_status hla_profile_enable(int32_t on) {
  g_msg[0] = 0;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_prof_on = on != 0;
  return HLA_OK;
}

hla_status hla_profile_read(float* ms_out, int32_t* launches_out, int32_t reset) {
  g_msg[0] = 0;
  HLA_CUDA(cudaDeviceSynchronize(), "hla_profile_read synchronize");
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (const StagePair& p : g_prof_pending) {
    float ms = 0.0f;
    if (cudaEventElapsedTime(&ms, p.a, p.b) == cudaSuccess) g_prof_ms[p.stage] += ms;
    cudaEventDestroy(p.a);
    cudaEventDestroy(p.b);
  }
  g_prof_pending.clear();
  for (int i = 0; i < HLA_STAGE_COUNT; ++i) {
    if (ms_out) ms_out[i] = (float)g_prof_ms[i];
    if (launches_out) launches_out[i] = (int32_t)g_prof_launches[i];
    if (reset) {
      g_prof_ms[i] = 0.0;
      g_prof_launches[i] = 0;
    }
  }
  return HLA_OK;
}

hla_status hla_check_bounded_wait(uint32_t limit_us, int32_t complete, hla_stream_t stream) {
  g_msg[0] = 0;
  if (limit_us < 1 || limit_us > 100000) return fail(HLA_ERR_INVALID_ARG, "limit_us must be in [1, 100000]");
  HLA_CUDA(hla::launch_wait_check((uint64_t)limit_us * 1000ull, complete != 0, (cudaStream_t)stream),
           "bounded-wait check launch");
  return HLA_OK;
}

hla_status hla_device_status(int32_t clear, uint32_t* code_out) {
  g_msg[0] = 0;
  HLA_CUDA(cudaDeviceSynchronize(), "hla_device_status synchronize");
  unsigned int word = 0, w = 0;
  HLA_CUDA(hla::read_error_word_decode(&w, clear != 0), "hla_device_status read");
  word |= w;
  HLA_CUDA(hla::read_error_word_compose_tc(&w, clear != 0), "hla_device_status read");
  word |= w;
  HLA_CUDA(hla::read_error_word_decode_stream(&w, clear != 0), "hla_device_status read");
  word |= w;
  HLA_CUDA(hla::read_error_word_transitions_tc(&w, clear != 0), "hla_device_status read");
  word |= w;
  HLA_CUDA(hla::read_error_word_readout_tc(&w, clear != 0), "hla_device_status read");
  word |= w;
  HLA_CUDA(hla::read_error_word_wait_check(&w, clear != 0), "hla_device_status read");
  word |= w;
  HLA_CUDA(hla::read_error_word_chain_tc(&w, clear != 0), "hla_device_status read");
  word |= w;
  HLA_CUDA(hla::read_error_word_chan_prep(&w, clear != 0), "hla_device_status read");
  word |= w;
  if (code_out) *code_out = word;
  if (word & (hla::kErrMbarTimeout | hla::kErrTmemAlloc))
    return fail(HLA_ERR_TIMEOUT, "a bounded device wait expired (code 0x%x)", word);
  if (word & hla::kErrCacheFull) return fail(HLA_ERR_WORKSPACE, "a decode step found the cache full (code 0x%x)", word);
  if (word & hla::kErrDecayRange)
    return fail(HLA_ERR_UNSUPPORTED,
                "a channel decayed below e^-80 within one 64-token sub-chunk: outside the range of the "
                "tensor-core channel-decay path (code 0x%x)",
                word);
  return HLA_OK;
}

}  // extern "C"
