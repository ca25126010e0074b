// Decode step kernels (one new token per sequence) and the prefill -> cache hand-off.
//
// HLA summary page, "Key Contributions" 3 (dynamic autoregressive decoding) and
// "Methodology in Plain English" paras. 3-4.  For the open chunk holding m tokens
// (the new one included), the output is o = S_t q with
//   S_t = S_in A_p + B_p,  S_in = gated composition over the active closed chunks,
// where (A_p, B_p) is the open chunk's own transition.  It is evaluated without
// forming any d x d product:
//   (1) right-to-left sweep over the open chunk's tokens gives x = A_p q and
//       y0 = B_p q:  c = k_t . x;  y0 += beta_t c v_t;  x <- alpha_t (x - beta_t c k_t);
//   (2) S_in x = sum_j g_j B_j prod_{l>j} ((1-g_l) I + g_l A_l) x, evaluated for the
//       active j in descending order:  y += g_j B_j x;  x <- (1-g_j) x + g_j A_j x;
//   (3) o = y + y0.
// Each active chunk's A_j and B_j are read exactly once; skipped chunks are not read.
#include "common.cuh"
#include "kernels.cuh"
#include "routing_recipe.cuh"

namespace hla {

HLA_DEFINE_ERROR_WORD(decode)

template <int D>
__device__ __forceinline__ float block_sum(float v, float* red) {
  // D threads, D/32 warps
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  const int w = threadIdx.x >> 5;
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  float s = 0.0f;
#pragma unroll
  for (int k = 0; k < D / 32; ++k) s += red[k];
  return s;
}

// grid B*H, block D.  Thread = channel / row.
template <int D, typename Tio>
__global__ void __launch_bounds__(128) decode_main_kernel(DecodeArgs a) {
  __shared__ __align__(16) float rq[D];
  __shared__ float xs[2][D];
  __shared__ float red[D / 32];
  __shared__ int wcount[D / 32];
  const int bh = blockIdx.x;
  const int b = bh / a.H;
  const int tid = threadIdx.x;
  const int C = a.C;
  const int n = a.n_chunks[b];
  const int m = a.m_partial[b];
  const int mp = m + 1;
  const long tok = (long)bh * D + tid;
  // (0) append the token to the open chunk
  const long bslot = ((long)bh * C + m) * D + tid;
  const Tio* qr_in = (const Tio*)(a.q_route ? a.q_route : a.q);
  const Tio* kr_in = (const Tio*)(a.k_route ? a.k_route : a.k);
  ((Tio*)a.buf_k)[bslot] = ((const Tio*)a.k)[tok];
  ((Tio*)a.buf_v)[bslot] = ((const Tio*)a.v)[tok];
  ((Tio*)a.buf_qr)[bslot] = qr_in[tok];
  ((Tio*)a.buf_kr)[bslot] = kr_in[tok];
  if (a.alpha_vec) a.buf_alpha[((long)bh * C + m) * D + tid] = a.alpha[(long)bh * D + tid];
  if (tid == 0) {
    if (!a.alpha_vec) a.buf_alpha[(long)bh * C + m] = a.alpha[bh];
    a.buf_beta[(long)bh * C + m] = a.beta[bh];
  }
  __syncthreads();
  const Tio* bk = (const Tio*)a.buf_k + (long)bh * C * D;
  const Tio* bv = (const Tio*)a.buf_v + (long)bh * C * D;
  // (1) open-chunk sweep
  float x = ldf((const Tio*)a.q + tok);
  float y0 = 0.0f;
  for (int t = mp - 1; t >= 0; --t) {
    const float kt = ldf(bk + (long)t * D + tid);
    const float c = block_sum<D>(kt * x, red);
    const float bt = a.buf_beta[(long)bh * C + t];
    // scalar decay, or this channel's decay
    const float at = a.alpha_vec ? a.buf_alpha[((long)bh * C + t) * D + tid] : a.buf_alpha[(long)bh * C + t];
    y0 = fmaf(bt * c, ldf(bv + (long)t * D + tid), y0);
    x = at * (x - bt * c * kt);
  }
  // (2) gates against every closed chunk, compacted ascending into the workspace
  int32_t* act_idx = a.act_idx + (long)bh * a.max_chunks;
  float* act_g = a.act_g + (long)bh * a.max_chunks;
  int cnt = 0;
  if (a.mode != HLA_GATES_ZERO && n > 0) {
    const route::Consts K = route::make_consts();
    if (a.mode == HLA_GATES_ROUTED) {
      // query pool over the open chunk's mp route tokens (channel = tid)
      const Tio* bq = (const Tio*)a.buf_qr + (long)bh * C * D + tid;
      const float inv_tau = __fdiv_rn(1.0f, a.tau);
      float mx = __fmul_rn(ldf(bq), inv_tau);
      for (int t = 1; t < mp; ++t) mx = fmaxf(mx, __fmul_rn(ldf(bq + (long)t * D), inv_tau));
      float s = 0.0f;
      for (int t = 0; t < mp; ++t)
        s = __fadd_rn(s, route::rexp(route::pool_shift(ldf(bq + (long)t * D), inv_tau, mx), K));
      rq[tid] = __fmul_rn(a.tau, __fadd_rn(mx, route::rlog(__fdiv_rn(s, (float)mp), K)));
      __syncthreads();
    }
    const int W = a.win > 0 ? a.win : 1;
    const float* rk = a.rk + (long)bh * a.max_chunks * W * D;
    for (int jb = 0; jb < n; jb += D) {
      const int j = jb + tid;
      float g = 1.0f;
      bool keep = false;
      if (j < n) {
        if (a.mode == HLA_GATES_ROUTED && a.win > 0) {
          // log-sum-exp over the closed chunk's window representatives
          float t[kMaxWindows];
          const float m = route::window_scores(rq, rk + (long)j * W * D, a.win, D, a.c_d, t);
          g = route::gate_from_window_scores(t, a.win, m, a.bias, K);
        } else if (a.mode == HLA_GATES_ROUTED) {
          const float* rkj = rk + (long)j * D;
          float dot = 0.0f;
          for (int c = 0; c < D; ++c) dot = route::dot_step(dot, rq[c], rkj[c]);
          g = route::gate_from_dot(dot, a.c_d, a.bias, K);
        }
        keep = a.thr <= 0.0f || g >= a.thr;
      }
      const unsigned int bal = __ballot_sync(0xFFFFFFFFu, keep);
      const int w = tid >> 5;
      if ((tid & 31) == 0) wcount[w] = __popc(bal);
      __syncthreads();
      int before = 0, total = 0;
      for (int k2 = 0; k2 < D / 32; ++k2) {
        if (k2 < w) before += wcount[k2];
        total += wcount[k2];
      }
      if (keep) {
        const int pos = cnt + before + __popc(bal & ((1u << (tid & 31)) - 1u));
        act_idx[pos] = j;
        act_g[pos] = g;
      }
      cnt += total;
      __syncthreads();
    }
  }
  // (3) backward chain over active chunks, descending j
  float y = 0.0f;
  int cur = 0;
  xs[0][tid] = x;
  __syncthreads();
  for (int p = cnt - 1; p >= 0; --p) {
    const int j = act_idx[p];
    const float g = act_g[p];
    const Tio* A = (const Tio*)a.A + ((long)bh * a.max_chunks + j) * (long)D * D + (long)tid * D;
    const Tio* Bm = (const Tio*)a.Bm + ((long)bh * a.max_chunks + j) * (long)D * D + (long)tid * D;
    float ax = 0.0f, bx = 0.0f;
#pragma unroll 8
    for (int c = 0; c < D; ++c) {
      const float xc = xs[cur][c];
      ax = fmaf(ldf(A + c), xc, ax);
      bx = fmaf(ldf(Bm + c), xc, bx);
    }
    y = fmaf(g, bx, y);
    xs[cur ^ 1][tid] = (1.0f - g) * xs[cur][tid] + g * ax;
    cur ^= 1;
    __syncthreads();
  }
  stf((Tio*)a.o + tok, y + y0);
}

// Key pool of the closing chunk into the cache (only sequences whose open chunk
// becomes full this step).  grid B*H, block D.
template <int D, typename Tio>
__device__ __forceinline__ void close_pool(const DecodeArgs& a) {
  const int bh = blockIdx.x;
  const int b = bh / a.H;
  const int tid = threadIdx.x;
  if (a.m_partial[b] + 1 != a.C) return;
  const int n = a.n_chunks[b];
  if (n >= a.max_chunks) {
    if (tid == 0) report_device_error(kErrCacheFull);
    return;
  }
  const route::Consts K = route::make_consts();
  const float inv_tau = __fdiv_rn(1.0f, a.tau);
  // one pool over the chunk, or one per window of C / W tokens
  const int W = a.win > 0 ? a.win : 1;
  const int len = a.C / W;
  for (int u = 0; u < W; ++u) {
    const Tio* bk = (const Tio*)a.buf_kr + ((long)bh * a.C + (long)u * len) * D + tid;
    float mx = __fmul_rn(ldf(bk), inv_tau);
    for (int t = 1; t < len; ++t) mx = fmaxf(mx, __fmul_rn(ldf(bk + (long)t * D), inv_tau));
    float s = 0.0f;
    for (int t = 0; t < len; ++t)
      s = __fadd_rn(s, route::rexp(route::pool_shift(ldf(bk + (long)t * D), inv_tau, mx), K));
    a.rk[(((long)bh * a.max_chunks + n) * W + u) * D + tid] =
        __fmul_rn(a.tau, __fadd_rn(mx, route::rlog(__fdiv_rn(s, (float)len), K)));
  }
}

// Launched as the closing transition's programmatic dependent: the two read the same
// open-chunk rows and counters and write disjoint outputs, so they may overlap.  Every
// CTA waits for the transition grid before it exits, so this grid completes after it;
// the counters kernel (this grid's dependent) waits for this grid alone.
template <int D, typename Tio>
__global__ void decode_close_pool_kernel(DecodeArgs a) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  close_pool<D, Tio>(a);
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

__global__ void decode_counters_kernel(int B, int C, int max_chunks, int32_t* n_chunks, int32_t* m_partial) {
  // the pool kernel (and through it the closing transition) read the counters
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  const int m = m_partial[b] + 1;
  if (m == C) {
    if (n_chunks[b] < max_chunks) n_chunks[b] += 1;
    m_partial[b] = 0;
  } else {
    m_partial[b] = m;
  }
}

// Prefill -> cache hand-off: copies the closed chunks' key pools (computed into the
// prefill workspace with chunk stride N) and the final partial chunk's tokens, and
// sets the counters.  grid B*H, block 128.
struct FillArgs {
  int B, H, T, C, d, N, max_chunks;
  int W;               // key representatives per chunk
  const float* rk_ws;  // [B,H,N*W,d]
  const void *qr, *kr, *k, *v;  // [B,T,H,d]
  const float *alpha, *beta;    // [B,T,H]
};

template <typename Tio>
__global__ void cache_fill_kernel(DecodeArgs c, FillArgs f) {
  const int bh = blockIdx.x;
  const int b = bh / f.H, h = bh % f.H;
  const int nc = f.T / f.C;
  const int m = f.T - nc * f.C;
  for (long idx = threadIdx.x; idx < (long)nc * f.W * f.d; idx += blockDim.x)
    c.rk[(long)bh * f.max_chunks * f.W * f.d + idx] = f.rk_ws[(long)bh * f.N * f.W * f.d + idx];
  const long HD = (long)f.H * f.d;
  for (long idx = threadIdx.x; idx < (long)m * f.d; idx += blockDim.x) {
    const int t = (int)(idx / f.d), ch = (int)(idx - (long)t * f.d);
    const long src = ((long)b * f.T + nc * f.C + t) * HD + (long)h * f.d + ch;
    const long dst = ((long)bh * f.C + t) * f.d + ch;
    ((Tio*)c.buf_k)[dst] = ((const Tio*)f.k)[src];
    ((Tio*)c.buf_v)[dst] = ((const Tio*)f.v)[src];
    ((Tio*)c.buf_qr)[dst] = ((const Tio*)f.qr)[src];
    ((Tio*)c.buf_kr)[dst] = ((const Tio*)f.kr)[src];
  }
  for (int t = threadIdx.x; t < m; t += blockDim.x) {
    const long src = ((long)b * f.T + nc * f.C + t) * f.H + h;
    if (!c.alpha_vec) c.buf_alpha[(long)bh * f.C + t] = f.alpha[src];
    c.buf_beta[(long)bh * f.C + t] = f.beta[src];
  }
  if (c.alpha_vec)  // channel-wise decay: alpha [B,T,H,d] into [B,H,C,d]
    for (long idx = threadIdx.x; idx < (long)m * f.d; idx += blockDim.x) {
      const int t = (int)(idx / f.d), ch = (int)(idx - (long)t * f.d);
      c.buf_alpha[((long)bh * f.C + t) * f.d + ch] = f.alpha[(((long)b * f.T + nc * f.C + t) * f.H + h) * f.d + ch];
    }
  if (h == 0 && threadIdx.x == 0) {
    c.n_chunks[b] = nc;
    c.m_partial[b] = m;
  }
}

// Prefill -> factored cache: K (from the input), Wb and Ub (bf16, from the
// transition kernel's workspace output) and the scales of every complete chunk.
// One CTA per (b, h, complete chunk), 16-byte copies.
__global__ void __launch_bounds__(256) factor_fill_kernel(FactorFillArgs f) {
  constexpr int C = 64, D = 128, PAD = C + 4;
  const long chunk = blockIdx.x;
  const int i = (int)(chunk % f.Nc);
  const long bh = chunk / f.Nc;
  const int b = (int)(bh / f.H), h = (int)(bh % f.H);
  const uint4* wb = (const uint4*)f.Wb + (bh * f.N + i) * (C * D / 8);
  const uint4* ub = (const uint4*)f.Ub + (bh * f.N + i) * (C * D / 8);
  const long slot = bh * f.max_chunks + i;
  uint4* kf = (uint4*)f.Kf + slot * (C * D / 8);
  uint4* wf = (uint4*)f.Wf + slot * (C * D / 8);
  uint4* uf = (uint4*)f.Uf + slot * (C * D / 8);
  for (int e = threadIdx.x; e < C * D / 8; e += blockDim.x) {
    const int t = e / (D / 8), c8 = e % (D / 8);
    const long src = (((long)b * f.T + (long)i * C + t) * f.H + h) * (D / 8) + c8;
    kf[e] = ((const uint4*)f.k)[src];
    wf[e] = wb[e];
    uf[e] = ub[e];
  }
  const float* ell = f.ell + (bh * f.N + i) * C;
  float* dfo = f.df + slot * PAD;
  const int tid = threadIdx.x;
  if (tid < C) dfo[tid] = expf(ell[C - 1] - ell[tid]);
  if (tid >= C && tid < PAD) dfo[tid] = tid == C ? expf(ell[C - 1]) : 0.0f;
}

cudaError_t launch_factor_fill(const FactorFillArgs& f, cudaStream_t s) {
  const long blocks = (long)f.B * f.H * f.Nc;
  if (blocks <= 0) return cudaSuccess;
  factor_fill_kernel<<<(unsigned)blocks, 256, 0, s>>>(f);
  return cudaGetLastError();
}

template <int D, typename Tio>
static cudaError_t launch_main(const DecodeArgs& a, cudaStream_t s) {
  decode_main_kernel<D, Tio><<<a.B * a.H, D, 0, s>>>(a);
  return cudaGetLastError();
}

template <int D, typename Tio>
static cudaError_t launch_close(const DecodeArgs& a, cudaStream_t s) {
  // close full chunks: transition into the cache, then the key pool, then counters
  TransArgs t{};
  t.B = a.B;
  t.H = a.H;
  t.T = a.C;
  t.C = a.C;
  t.d = D;
  t.dtype = a.dtype;
  t.in.k = a.buf_k;
  t.in.v = a.buf_v;
  t.in.alpha = a.buf_alpha;
  t.in.beta = a.buf_beta;
  t.in.sb = (long)a.H * a.C * D;
  t.in.sh = (long)a.C * D;
  t.in.st = D;
  t.in.ab = (long)a.H * a.C;
  t.in.ah = a.C;
  t.in.at = 1;
  if (a.alpha_vec) {  // buf_alpha [B,H,C,d]: the alpha strides are those of beta times d
    t.in.ab *= D;
    t.in.ah *= D;
    t.in.at *= D;
    t.in.alpha_vec = 1;
  }
  t.n_chunks = 1;
  t.A = const_cast<void*>(a.A);
  t.Bm = const_cast<void*>(a.Bm);
  t.Kf = a.Kf;  // factored cache: the transition kernel writes the factors instead of A/B
  t.Wf = a.Wf;
  t.Uf = a.Uf;
  t.df = a.df;
  t.ab_chunk_stride = a.max_chunks;
  t.ab_chunk_offset = 0;
  t.close_m = a.m_partial;
  t.close_n = a.n_chunks;
  // the transition kernel never writes past max_chunks; the pool kernel flags it.
  // Chunks longer than one 64-token WY tile close by the token rule (no workspace).
  cudaError_t e = (a.C > 64 || a.alpha_vec) ? launch_transitions_token(t, s) : launch_transitions(t, s);
  if (e != cudaSuccess) return e;
  // the pool and counters kernels are programmatic dependents of the kernel before each
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.B * a.H);
  cfg.blockDim = dim3(D);
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, decode_close_pool_kernel<D, Tio>, a);
  if (e != cudaSuccess) return e;
  cfg.gridDim = dim3((a.B + 127) / 128);
  cfg.blockDim = dim3(128);
  e = cudaLaunchKernelEx(&cfg, decode_counters_kernel, a.B, a.C, a.max_chunks, a.n_chunks, a.m_partial);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_decode_main(const DecodeArgs& a, cudaStream_t s) {
  if (a.format == HLA_CACHE_FACTORED) return launch_decode_stream_factored(a, s);
  if (a.d == 128 && a.dtype == HLA_BF16) return launch_decode_stream(a, s);
  if (a.d == 128) return a.dtype == HLA_BF16 ? launch_main<128, __nv_bfloat16>(a, s) : launch_main<128, float>(a, s);
  return a.dtype == HLA_BF16 ? launch_main<64, __nv_bfloat16>(a, s) : launch_main<64, float>(a, s);
}

cudaError_t launch_decode_close(const DecodeArgs& a, cudaStream_t s) {
  if (a.d == 128)
    return a.dtype == HLA_BF16 ? launch_close<128, __nv_bfloat16>(a, s) : launch_close<128, float>(a, s);
  return a.dtype == HLA_BF16 ? launch_close<64, __nv_bfloat16>(a, s) : launch_close<64, float>(a, s);
}

cudaError_t launch_cache_fill(const DecodeArgs& c, const float* rk_ws, const void* q_route, const void* k_route,
                              const void* k, const void* v, const float* alpha, const float* beta, int T,
                              cudaStream_t s) {
  FillArgs f{};
  f.B = c.B;
  f.H = c.H;
  f.T = T;
  f.C = c.C;
  f.d = c.d;
  f.N = (T + c.C - 1) / c.C;
  f.max_chunks = c.max_chunks;
  f.W = c.win > 0 ? c.win : 1;
  f.rk_ws = rk_ws;
  f.qr = q_route;
  f.kr = k_route;
  f.k = k;
  f.v = v;
  f.alpha = alpha;
  f.beta = beta;
  if (c.dtype == HLA_BF16)
    cache_fill_kernel<__nv_bfloat16><<<c.B * c.H, 128, 0, s>>>(c, f);
  else
    cache_fill_kernel<float><<<c.B * c.H, 128, 0, s>>>(c, f);
  return cudaGetLastError();
}

}  // namespace hla
