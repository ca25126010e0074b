// Routing kernels: per-chunk log-mean-exp pools, gates and compacted active lists.
// Built with -fmad=false; the recipe's products and sums are __f*_rn intrinsics or
// explicit fused multiply-adds.
#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"
#include "routing_recipe.cuh"

namespace hla {

// ---------------------------------------------------------------------------
// Pools.  grid (N, B, 2 * groups), 64 threads; blockIdx.z = tensor * groups + group,
// a group is 128 consecutive channels of the H*d channel row and a thread owns two
// adjacent channels of one chunk.  For a fixed token the H*d channels are
// contiguous, so every token row is read coalesced.  bf16 inputs are read once
// into registers (one bf16 pair per token); float32 inputs are read twice (the
// second pass hits L1/L2).
//   max:  multiplying by 1/tau > 0 is monotone under rounding, so
//         max_t fl(x_t * (1/tau)) = fl((max_t x_t) * (1/tau)): one multiply per
//         channel.
//   sum:  s = sum_t exp(fma(x_t, 1/tau, -m)) in ascending t; the two channels
//         of a thread go through packed float32 pairs.
// out index: ((b*H + h)*out_chunk_stride + c)*d + ch.
// ---------------------------------------------------------------------------

namespace {
constexpr int kPoolBlock = 16;  // tokens read per step by the pools

// The recipe's e^x on a pair of values with packed float32 arithmetic
// (sm_100; each lane of __ffma2_rn / __fadd2_rn / __fmul2_rn is rounded as its
// scalar counterpart).  Every product that feeds a sum is a fused multiply-add in
// the recipe itself, because the code generator contracts a packed multiply that
// feeds a packed add; the product p * 2^n that the caller adds to its sum is exact,
// so contracting it changes no bit.
//   kInRange = true:  both inputs in [-86, 88] (the bits of route::rexp_core);
//   kInRange = false: inputs <= 0, those below -86 give 0 (route::rexp_nonpos).
template <bool kInRange>
__device__ __forceinline__ float2 rexp2(float2 x, const route::Consts& k) {
  const float2 xc = kInRange ? x : make_float2(fmaxf(x.x, -86.0f), fmaxf(x.y, -86.0f));
  const float2 sum = __ffma2_rn(xc, make_float2(k.log2e, k.log2e), make_float2(route::kRoundMagic, route::kRoundMagic));
  const float2 n = __fadd2_rn(sum, make_float2(-route::kRoundMagic, -route::kRoundMagic));
  const float2 nn = make_float2(-n.x, -n.y);
  const float2 r = __ffma2_rn(nn, make_float2(k.ln2_lo, k.ln2_lo), __ffma2_rn(nn, make_float2(k.ln2_hi, k.ln2_hi), xc));
  float2 p = make_float2((float)(1.0 / 5040.0), (float)(1.0 / 5040.0));
  p = __ffma2_rn(p, r, make_float2((float)(1.0 / 720.0), (float)(1.0 / 720.0)));
  p = __ffma2_rn(p, r, make_float2((float)(1.0 / 120.0), (float)(1.0 / 120.0)));
  p = __ffma2_rn(p, r, make_float2((float)(1.0 / 24.0), (float)(1.0 / 24.0)));
  p = __ffma2_rn(p, r, make_float2((float)(1.0 / 6.0), (float)(1.0 / 6.0)));
  p = __ffma2_rn(p, r, make_float2(0.5f, 0.5f));
  p = __ffma2_rn(p, r, make_float2(1.0f, 1.0f));
  p = __ffma2_rn(p, r, make_float2(1.0f, 1.0f));
  const float2 sc = make_float2(__uint_as_float((__float_as_uint(sum.x) << 23) + route::kScaleOffset),
                                __uint_as_float((__float_as_uint(sum.y) << 23) + route::kScaleOffset));
  const float2 e = __fmul2_rn(p, sc);
  if (kInRange) return e;
  return make_float2(x.x < -86.0f ? 0.0f : e.x, x.y < -86.0f ? 0.0f : e.y);
}

// Lane-wise maximum / minimum of two bf16 pairs (exact).
__device__ __forceinline__ uint32_t bf16x2_max(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t bf16x2_min(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("min.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// route::gate_from_dot on a pair of dot products: z = fma(dot, c_d, b), then
// 1 / (1 + exp(-z)) with the exp's range checks (-z > 88 -> +inf, -z < -86 -> 0).
__device__ __forceinline__ float2 gate2_from_dot(float2 dot, float c_d, float bias, const route::Consts& k) {
  const float2 z = __ffma2_rn(dot, make_float2(c_d, c_d), make_float2(bias, bias));
  const float2 x = make_float2(-z.x, -z.y);
  const float2 xc = make_float2(fminf(fmaxf(x.x, -86.0f), 88.0f), fminf(fmaxf(x.y, -86.0f), 88.0f));
  float2 e = rexp2<true>(xc, k);
  e.x = x.x > 88.0f ? CUDART_INF_F : (x.x < -86.0f ? 0.0f : e.x);
  e.y = x.y > 88.0f ? CUDART_INF_F : (x.y < -86.0f ? 0.0f : e.y);
  const float2 den = __fadd2_rn(make_float2(1.0f, 1.0f), e);
  return make_float2(__frcp_rn(den.x), __frcp_rn(den.y));
}

// s += exp(fma(x_t, inv_tau, -m)) over the bf16 pairs of tokens t0 .. t0+15 (t < n),
// ascending t, read again from global memory (L1 / L2 hits: the first pass read them).
template <bool kInRange>
__device__ __forceinline__ float2 pool_sum_bf16(float2 s, const uint32_t* colw, size_t stride, int t0, int n,
                                                float inv_tau, float m0, float m1, const route::Consts& K) {
  uint32_t w[kPoolBlock];
#pragma unroll
  for (int t = 0; t < kPoolBlock; ++t) w[t] = t0 + t < n ? __ldg(colw + (size_t)(t0 + t) * stride) : 0u;
#pragma unroll
  for (int t = 0; t < kPoolBlock; ++t)
    if (t0 + t < n) {
      const float2 u = __ffma2_rn(make_float2(__uint_as_float(w[t] << 16), __uint_as_float(w[t] & 0xFFFF0000u)),
                                  make_float2(inv_tau, inv_tau), make_float2(-m0, -m1));
      s = __fadd2_rn(s, rexp2<kInRange>(u, K));
    }
  return s;
}
}  // namespace

constexpr int kPoolMaxC = 256;  // longest chunk (or window) pooled

template <typename Tin>
__global__ void __launch_bounds__(64, 16) pool_kernel(const Tin* __restrict__ x0, const Tin* __restrict__ x1,
                                                  float* __restrict__ r0, float* __restrict__ r1, int T, int H,
                                                  int d, int C, int out_chunk_stride, float tau) {
  constexpr bool kBf16 = sizeof(Tin) == 2;
  const int groups = (H * d + 127) / 128;
  const int c = blockIdx.x;
  const int b = blockIdx.y;
  const int which = blockIdx.z / groups;
  const int grp = blockIdx.z - which * groups;
  const Tin* x = which == 0 ? x0 : x1;
  float* r = which == 0 ? r0 : r1;
  if (x == nullptr || r == nullptr) return;
  const int HD = H * d;
  const int ch0 = grp * 128 + 2 * threadIdx.x;
  if (ch0 >= HD) return;
  const route::Consts K = route::make_consts();
  const float inv_tau = __fdiv_rn(1.0f, tau);
  const int t0 = c * C;
  const int n = min(C, T - t0);
  // window representatives of a final partial chunk may start past the sequence: such
  // windows are never read (only complete chunks are keys), so nothing is pooled
  if (n <= 0) return;
  const Tin* col = x + ((size_t)b * T + t0) * HD + ch0;
  float s0 = 0.0f, s1 = 0.0f, m0, m1;
  if constexpr (kBf16) {
    // H*d and ch0 are even, so each bf16 pair is one aligned 32-bit word.  Two passes
    // over the chunk, 16 tokens at a time (few registers, so the pools can share the
    // SMs with a concurrent kernel): the extremes, then the sum of exponentials.
    const uint32_t* colw = reinterpret_cast<const uint32_t*>(col);
    const size_t stride = (size_t)HD / 2;
    uint32_t hi = __ldg(colw), lo = hi;
    for (int t0 = 0; t0 < n; t0 += kPoolBlock) {
      uint32_t w[kPoolBlock];
#pragma unroll
      for (int t = 0; t < kPoolBlock; ++t) w[t] = t0 + t < n ? __ldg(colw + (size_t)(t0 + t) * stride) : hi;
#pragma unroll
      for (int t = 0; t < kPoolBlock; ++t) {
        hi = bf16x2_max(hi, w[t]);
        lo = bf16x2_min(lo, w[t]);
      }
    }
    m0 = __fmul_rn(__uint_as_float(hi << 16), inv_tau);
    m1 = __fmul_rn(__uint_as_float(hi & 0xFFFF0000u), inv_tau);
    // fma is monotone in x (1/tau > 0), so the smallest shifted value comes from the
    // smallest input; when it is >= -86 no exp of the chunk needs the range checks
    const bool in_range = __fmaf_rn(__uint_as_float(lo << 16), inv_tau, -m0) >= -86.0f &&
                          __fmaf_rn(__uint_as_float(lo & 0xFFFF0000u), inv_tau, -m1) >= -86.0f;
    float2 ss = make_float2(0.0f, 0.0f);
    for (int t0 = 0; t0 < n; t0 += kPoolBlock)
      ss = in_range ? pool_sum_bf16<true>(ss, colw, stride, t0, n, inv_tau, m0, m1, K)
                    : pool_sum_bf16<false>(ss, colw, stride, t0, n, inv_tau, m0, m1, K);
    s0 = ss.x;
    s1 = ss.y;
  } else {
    const float2* colf = reinterpret_cast<const float2*>(col);
    const size_t stride = (size_t)HD / 2;
    float2 v = colf[0];
    float a0 = v.x, a1 = v.y;
    for (int t = 1; t < n; ++t) {
      v = colf[t * stride];
      a0 = fmaxf(a0, v.x);
      a1 = fmaxf(a1, v.y);
    }
    m0 = __fmul_rn(a0, inv_tau);
    m1 = __fmul_rn(a1, inv_tau);
    for (int t = 0; t < n; ++t) {
      v = colf[t * stride];
      s0 = __fadd_rn(s0, route::rexp_nonpos(route::pool_shift(v.x, inv_tau, m0), K));
      s1 = __fadd_rn(s1, route::rexp_nonpos(route::pool_shift(v.y, inv_tau, m1), K));
    }
  }
  const float v0 = __fmul_rn(tau, __fadd_rn(m0, route::rlog(__fdiv_rn(s0, (float)n), K)));
  const float v1 = __fmul_rn(tau, __fadd_rn(m1, route::rlog(__fdiv_rn(s1, (float)n), K)));
  const int h = ch0 / d;
  const int cc = ch0 - h * d;  // d is even, so both channels share the head
  float* out = r + (((size_t)b * H + h) * out_chunk_stride + c) * d + cc;
  out[0] = v0;
  out[1] = v1;
}

// ---------------------------------------------------------------------------
// Pools of bf16 inputs with chunks of up to 64 tokens, staged through shared memory.
// A unit is (tensor, b, chunk, group of 64 channels): a tile of n <= 64 token rows of
// 128 bytes.  Each warp walks units with a grid-wide stride and keeps two tile
// buffers: the next unit's rows are in flight (16-byte cp.async, one 128-byte row
// per 8 lanes) while the current one is reduced, lane = two adjacent channels.  The
// arithmetic, and so every bit, is that of pool_kernel.
// ---------------------------------------------------------------------------
constexpr int kTileWarps = 4;
constexpr int kTileRows = 64;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

struct PoolTileArgs {
  const __nv_bfloat16* x[2];
  float* r[2];
  int B, T, H, d, C, N, out_chunk_stride, groups;
  long units;
  float tau;
};

__device__ __forceinline__ void pool_tile_fetch(const PoolTileArgs& a, long u, uint32_t buf, int lane, int& n) {
  const int g = (int)(u % a.groups);
  long r = u / a.groups;
  const int c = (int)(r % a.N);
  r /= a.N;
  const int b = (int)(r % a.B);
  const int which = (int)(r / a.B);
  const int t0 = c * a.C;
  n = min(a.C, a.T - t0);
  const long HD = (long)a.H * a.d;
  const __nv_bfloat16* x = which == 0 ? a.x[0] : a.x[1];
  const char* src = (const char*)(x + ((long)b * a.T + t0) * HD + g * 64) + (lane & 7) * 16;
  for (int t = lane >> 3; t < n; t += 4) cp_async16(buf + t * 128 + (lane & 7) * 16, src + (long)t * HD * 2);
  asm volatile("cp.async.commit_group;" ::: "memory");
}

__global__ void __launch_bounds__(32 * kTileWarps) pool_tile_kernel(PoolTileArgs a) {
  extern __shared__ __align__(16) uint8_t pool_sm[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t base = (uint32_t)__cvta_generic_to_shared(pool_sm) + warp * 2 * kTileRows * 128;
  const uint32_t* words = reinterpret_cast<const uint32_t*>(pool_sm + warp * 2 * kTileRows * 128);
  const long stride = (long)gridDim.x * kTileWarps;
  long u = (long)blockIdx.x * kTileWarps + warp;
  if (u >= a.units) return;
  const route::Consts K = route::make_consts();
  const float inv_tau = __fdiv_rn(1.0f, a.tau);
  int n_cur = 0, n_next = 0;
  pool_tile_fetch(a, u, base, lane, n_cur);
  for (int k = 0; u < a.units; u += stride, ++k) {
    const int cur = k & 1;
    const bool more = u + stride < a.units;
    if (more) {
      pool_tile_fetch(a, u + stride, base + (cur ^ 1) * kTileRows * 128, lane, n_next);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncwarp();
    const uint32_t* w = words + cur * kTileRows * 32 + lane;
    const int n = n_cur;
    if (n <= 0) {
      // a window past the end of the sequence (a final partial chunk): never read
      n_cur = n_next;
      continue;
    }
    uint32_t hi = w[0], lo = hi;
    for (int t = 1; t < n; ++t) {
      hi = bf16x2_max(hi, w[t * 32]);
      lo = bf16x2_min(lo, w[t * 32]);
    }
    const float m0 = __fmul_rn(__uint_as_float(hi << 16), inv_tau);
    const float m1 = __fmul_rn(__uint_as_float(hi & 0xFFFF0000u), inv_tau);
    const bool in_range = __fmaf_rn(__uint_as_float(lo << 16), inv_tau, -m0) >= -86.0f &&
                          __fmaf_rn(__uint_as_float(lo & 0xFFFF0000u), inv_tau, -m1) >= -86.0f;
    float2 s = make_float2(0.0f, 0.0f);
    if (in_range) {
#pragma unroll 8
      for (int t = 0; t < n; ++t) {
        const uint32_t x = w[t * 32];
        const float2 v = __ffma2_rn(make_float2(__uint_as_float(x << 16), __uint_as_float(x & 0xFFFF0000u)),
                                    make_float2(inv_tau, inv_tau), make_float2(-m0, -m1));
        s = __fadd2_rn(s, rexp2<true>(v, K));
      }
    } else {
#pragma unroll 8
      for (int t = 0; t < n; ++t) {
        const uint32_t x = w[t * 32];
        const float2 v = __ffma2_rn(make_float2(__uint_as_float(x << 16), __uint_as_float(x & 0xFFFF0000u)),
                                    make_float2(inv_tau, inv_tau), make_float2(-m0, -m1));
        s = __fadd2_rn(s, rexp2<false>(v, K));
      }
    }
    __syncwarp();  // every lane has read the buffer before the next fetch refills it
    const float v0 = __fmul_rn(a.tau, __fadd_rn(m0, route::rlog(__fdiv_rn(s.x, (float)n), K)));
    const float v1 = __fmul_rn(a.tau, __fadd_rn(m1, route::rlog(__fdiv_rn(s.y, (float)n), K)));
    const int g = (int)(u % a.groups);
    long r = u / a.groups;
    const int c = (int)(r % a.N);
    r /= a.N;
    const int b = (int)(r % a.B);
    const int which = (int)(r / a.B);
    const int ch = g * 64 + 2 * lane;
    const int h = ch / a.d, cc = ch - h * a.d;
    float* out = which == 0 ? a.r[0] : a.r[1];
    *reinterpret_cast<float2*>(out + (((long)b * a.H + h) * a.out_chunk_stride + c) * a.d + cc) = make_float2(v0, v1);
    n_cur = n_next;
  }
}

// ---------------------------------------------------------------------------
// Gates + active lists.  One warp per query-chunk row (b, h, i).  Lane j' handles
// j = jb + lane; the dot product runs over channels in ascending order.  Active j
// (ascending) are compacted with a warp ballot.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) gates_kernel(GatesArgs a) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int rows = a.B * a.H * a.N;
  if (warp >= rows) return;
  const int i = warp % a.N;
  const int bh = warp / a.N;
  const route::Consts K = route::make_consts();
  const float* rq = a.rq + ((size_t)bh * a.N + i) * a.d;
  const int W = a.win > 0 ? a.win : 1;
  const float* rk = a.rk + (size_t)bh * a.N * W * a.d;
  const size_t row = (size_t)warp * a.N;
  int cnt = 0;
  for (int jb = 0; jb < a.N; jb += 32) {
    const int j = jb + lane;
    float g = 0.0f;
    const bool valid = j < i;
    if (valid) {
      if (a.mode == HLA_GATES_ROUTED && a.win > 0) {
        // log-sum-exp over the key chunk's window representatives
        float t[kMaxWindows];
        const float m = route::window_scores(rq, rk + (size_t)j * W * a.d, a.win, a.d, a.c_d, t);
        g = route::gate_from_window_scores(t, a.win, m, a.bias, K);
      } else if (a.mode == HLA_GATES_ROUTED) {
        const float* rkj = rk + (size_t)j * a.d;
        float dot = 0.0f;
        for (int c = 0; c < a.d; ++c) dot = route::dot_step(dot, rq[c], rkj[c]);
        g = route::gate_from_dot(dot, a.c_d, a.bias, K);
      } else if (a.mode == HLA_GATES_ONE) {
        g = 1.0f;
      } else if (a.mode == HLA_GATES_USER) {
        g = a.user_gates[row + j];
      }
    }
    const bool keep = valid && (a.thr <= 0.0f || g >= a.thr);
    const unsigned int bal = __ballot_sync(0xFFFFFFFFu, keep);
    if (keep) {
      const int pos = cnt + __popc(bal & ((1u << lane) - 1u));
      if (a.act_idx) a.act_idx[row + pos] = j;
      if (a.act_g) a.act_g[row + pos] = g;
    }
    if (a.gates_out && j < a.N) a.gates_out[row + j] = valid ? g : 0.0f;
    cnt += __popc(bal);
  }
  if (lane == 0 && a.act_cnt) a.act_cnt[warp] = cnt;
  if (a.active_cnt_out && lane == 0) a.active_cnt_out[warp] = cnt;
  if (a.pad_act_idx && a.act_idx) {
    for (int p = cnt + lane; p < a.N; p += 32) a.act_idx[row + p] = -1;
  }
  if (a.active_idx_out) {
    // copy the compacted row (ascending) and pad with -1
    __syncwarp();
    for (int p = lane; p < a.N; p += 32) a.active_idx_out[row + p] = p < cnt ? a.act_idx[row + p] : -1;
  }
}

// ---------------------------------------------------------------------------
// Routed gates, tiled: one CTA per (TI query chunks, b, h), 256 threads.  A thread
// computes 4 rows x CPT columns of a TI x 64 gate tile (TI = 64: 4 x 4; TI = 16,
// for grids too small to fill the GPU: 4 x 1).  Every dot product still runs over
// channels in ascending order, one fused multiply-add per channel, so the
// bits equal the per-pair recipe.  Active chunks are compacted row by row in
// ascending j.
// ---------------------------------------------------------------------------
template <int D, int TI>
__global__ void __launch_bounds__(256) gates_tiled_kernel(GatesArgs a) {
  constexpr int TJ = 64;
  constexpr int CPT = (TI * TJ) / (256 * 4);  // columns per thread
  constexpr int NTX = TJ / CPT;               // threads along j
  constexpr int QMASK = TI / 4 - 1;           // swizzle range of the rq tile
  constexpr int FILL_Q = (TI / 4) * D / 256;  // float4 stores per thread, rq tile
  constexpr int FILL_K = (TJ / 4) * D / 256;  // float4 stores per thread, rk tile
  static_assert(CPT == 1 || CPT == 4, "tile shape");
  static_assert(FILL_Q >= 1 && FILL_K >= 1, "tile shape");
  extern __shared__ float smf[];
  float(*rqT)[TI] = reinterpret_cast<float(*)[TI]>(smf);            // [D][TI] rq tile, channel-major
  float(*rkT)[TJ] = reinterpret_cast<float(*)[TJ]>(smf + D * TI);   // [D][TJ] rk tile, channel-major
  float(*G)[TJ + 1] = reinterpret_cast<float(*)[TJ + 1]>(smf + D * TI + D * TJ);  // [TI][TJ+1]
  int* cnt_s = reinterpret_cast<int*>(smf + D * TI + D * TJ + TI * (TJ + 1));      // [TI]
  // 1-D grid in descending row-tile order over all heads: the CTAs with the most key
  // tiles (the last query chunks) start first, the short ones fill the tail
  const int nrt = (a.N + TI - 1) / TI;
  const int BHn = a.B * a.H;
  const int i0 = (nrt - 1 - (int)(blockIdx.x / BHn)) * TI;
  const int bh = (int)(blockIdx.x % BHn);
  const int tid = threadIdx.x;
  const int ty = tid / NTX, tx = tid % NTX;
  const int warp = tid >> 5, lane = tid & 31;
  const route::Consts K = route::make_consts();
  const float* rq = a.rq + (size_t)bh * a.N * D;
  const float* rk = a.rk + (size_t)bh * a.N * D;
  // Tiles are channel-major with their float4 row groups XOR-swizzled by the channel
  // (group g of channel c at slot g ^ (c % groups)): the fill below (one channel,
  // four consecutive rows per thread, one 16-byte store) and the reads of the dot
  // products are free of bank conflicts.  All loads of a fill are issued before its
  // stores.
  {
    float4 v[FILL_Q];
#pragma unroll
    for (int f = 0; f < FILL_Q; ++f) {
      const int e = tid + 256 * f;
      const int g = e / D, c = e - g * D;
      float* vp = &v[f].x;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + 4 * g + u;
        vp[u] = i < a.N ? rq[(size_t)i * D + c] : 0.0f;
      }
    }
#pragma unroll
    for (int f = 0; f < FILL_Q; ++f) {
      const int e = tid + 256 * f;
      const int g = e / D, c = e - g * D;
      *(float4*)&rqT[c][(g ^ (c & QMASK)) << 2] = v[f];
    }
  }
  if (tid < TI) cnt_s[tid] = 0;
  const int i_last = min(a.N, i0 + TI) - 1;
  // rk tiles are software-pipelined: the next tile's loads are in flight while the
  // current tile is multiplied
  float4 v[FILL_K];
  auto load_rk = [&](int j0) {
#pragma unroll
    for (int f = 0; f < FILL_K; ++f) {
      const int e = tid + 256 * f;
      const int g = e / D, c = e - g * D;
      float* vp = &v[f].x;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int j = j0 + 4 * g + u;
        vp[u] = j < a.N ? rk[(size_t)j * D + c] : 0.0f;
      }
    }
  };
  if (i_last > 0) load_rk(0);
  for (int j0 = 0; j0 < i_last; j0 += TJ) {
    __syncthreads();  // the previous tile's readers are done
#pragma unroll
    for (int f = 0; f < FILL_K; ++f) {
      const int e = tid + 256 * f;
      const int g = e / D, c = e - g * D;
      *(float4*)&rkT[c][(g ^ (c & 15)) << 2] = v[f];
    }
    __syncthreads();
    if (j0 + TJ < i_last) load_rk(j0 + TJ);
    // accumulators of rows (2p, 2p + 1) and column w, packed as one float pair:
    // each lane of a packed fused multiply-add is rounded on its own
    float2 acc[2][CPT];
#pragma unroll
    for (int u = 0; u < 2; ++u)
#pragma unroll
      for (int w = 0; w < CPT; ++w) acc[u][w] = make_float2(0.0f, 0.0f);
#pragma unroll 4
    for (int c = 0; c < D; ++c) {
      const float4 q4 = *(const float4*)&rqT[c][(ty ^ (c & QMASK)) << 2];
      const float2 qv[2] = {make_float2(q4.x, q4.y), make_float2(q4.z, q4.w)};
      float kv[CPT];
      if constexpr (CPT == 4) {
        const float4 k4 = *(const float4*)&rkT[c][(tx ^ (c & 15)) << 2];
        kv[0] = k4.x;
        kv[1] = k4.y;
        kv[2] = k4.z;
        kv[3] = k4.w;
      } else {
        kv[0] = rkT[c][(((tx >> 2) ^ (c & 15)) << 2) | (tx & 3)];
      }
#pragma unroll
      for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int w = 0; w < CPT; ++w)
          acc[u][w] = __ffma2_rn(qv[u], make_float2(kv[w], kv[w]), acc[u][w]);
    }
#pragma unroll
    for (int u = 0; u < 2; ++u)
#pragma unroll
      for (int w = 0; w < CPT; ++w) {
        const float2 g = gate2_from_dot(acc[u][w], a.c_d, a.bias, K);
        G[ty * 4 + 2 * u][tx * CPT + w] = g.x;
        G[ty * 4 + 2 * u + 1][tx * CPT + w] = g.y;
      }
    __syncthreads();
    // compaction: warp w handles rows w, w+8, ...
    for (int r = warp; r < TI; r += 8) {
      const int i = i0 + r;
      if (i >= a.N) continue;
      const size_t row = ((size_t)bh * a.N + i) * a.N;
      int cnt = cnt_s[r];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int jj = hh * 32 + lane;
        const int j = j0 + jj;
        const bool valid = j < i;
        const float g = G[r][jj];
        const bool keep = valid && (a.thr <= 0.0f || g >= a.thr);
        const unsigned int bal = __ballot_sync(0xFFFFFFFFu, keep);
        if (keep) {
          const int pos = cnt + __popc(bal & ((1u << lane) - 1u));
          if (a.act_idx) a.act_idx[row + pos] = j;
          if (a.act_g) a.act_g[row + pos] = g;
        }
        if (a.gates_out && j < a.N) a.gates_out[row + j] = valid ? g : 0.0f;
        cnt += __popc(bal);
      }
      if (lane == 0) cnt_s[r] = cnt;
    }
  }
  __syncthreads();
  // counts, zero gates beyond the computed tiles, padding and copies
  for (int r = warp; r < TI; r += 8) {
    const int i = i0 + r;
    if (i >= a.N) continue;
    const size_t row = ((size_t)bh * a.N + i) * a.N;
    const int cnt = cnt_s[r];
    if (lane == 0) {
      if (a.act_cnt) a.act_cnt[(size_t)bh * a.N + i] = cnt;
      if (a.active_cnt_out) a.active_cnt_out[(size_t)bh * a.N + i] = cnt;
    }
    const int jdone = (i_last > 0) ? ((i_last + TJ - 1) / TJ) * TJ : 0;
    if (a.gates_out)
      for (int j = jdone + lane; j < a.N; j += 32) a.gates_out[row + j] = 0.0f;
    if (a.pad_act_idx && a.act_idx)
      for (int p = cnt + lane; p < a.N; p += 32) a.act_idx[row + p] = -1;
    if (a.active_idx_out) {
      __syncwarp();
      for (int p = lane; p < a.N; p += 32) a.active_idx_out[row + p] = p < cnt ? a.act_idx[row + p] : -1;
    }
  }
}

template <int D, int TI>
static cudaError_t launch_gates_tiled(const GatesArgs& a, cudaStream_t s) {
  const unsigned grid = (unsigned)(((a.N + TI - 1) / TI) * a.B * a.H);
  const size_t smem = (size_t)(D * TI + D * 64 + TI * 65 + TI) * 4;
  cudaError_t e = cudaFuncSetAttribute(gates_tiled_kernel<D, TI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  gates_tiled_kernel<D, TI><<<grid, 256, smem, s>>>(a);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Routed gates with window representatives, tiled: one CTA per (TI query chunks,
// b, h), 256 threads.  Key rows are the window pools (row j * W + u of chunk j);
// a tile holds 64 of them, i.e. 64 / W chunks.  Per tile:
//   1. TI x 64 window scores t = dot * c_d, each dot one fma chain over ascending
//      channels (TI / 4 chains per thread, key row fixed per thread);
//   2. one thread per (query chunk, key chunk) takes the log-sum-exp over its W
//      scores in ascending u and the sigmoid (the recipe of gate_from_window_scores);
//   3. warps compact each row's kept chunks in ascending j.
// Query and key tiles are row-major with one float of padding per row, so the key
// reads of a warp (32 different rows, one channel) fall in distinct banks.
// ---------------------------------------------------------------------------
template <int D, int TI>
__global__ void __launch_bounds__(256) gates_window_tiled_kernel(GatesArgs a) {
  constexpr int KR = 64;            // key rows (window pools) per tile
  constexpr int DP = D + 1;
  constexpr int CH = TI / 4;        // dot chains per thread
  extern __shared__ float smf[];
  float* rqS = smf;                         // [TI][DP]
  float* rkS = rqS + TI * DP;               // [KR][DP]
  float* Ts = rkS + KR * DP;                // [TI][KR]  scores
  float* Gs = Ts + TI * KR;                 // [TI][KR]  gates of the tile's chunks
  int* cnt_s = reinterpret_cast<int*>(Gs + TI * KR);  // [TI]
  const int W = a.win;
  const int JC = KR / W;                    // chunks per tile
  const int i0 = blockIdx.x * TI;
  const int bh = blockIdx.y;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const route::Consts K = route::make_consts();
  const float* rq = a.rq + (size_t)bh * a.N * D;
  const float* rk = a.rk + (size_t)bh * a.N * W * D;
  for (int e = tid; e < TI * D; e += 256) {
    const int r = e / D, c = e - r * D;
    rqS[r * DP + c] = i0 + r < a.N ? rq[(size_t)(i0 + r) * D + c] : 0.0f;
  }
  if (tid < TI) cnt_s[tid] = 0;
  const int i_last = min(a.N, i0 + TI) - 1;
  const int kr = tid & (KR - 1);            // key row of this thread
  const int qb = (tid >> 6) * CH;           // first query row of this thread
  for (int j0 = 0; j0 < i_last; j0 += JC) {
    __syncthreads();  // the previous tile's readers are done
    for (int e = tid; e < KR * D; e += 256) {
      const int r = e / D, c = e - r * D;
      const size_t row = (size_t)j0 * W + r;
      rkS[r * DP + c] = row < (size_t)a.N * W ? rk[row * D + c] : 0.0f;
    }
    __syncthreads();
    float acc[CH];
#pragma unroll
    for (int q = 0; q < CH; ++q) acc[q] = 0.0f;
#pragma unroll 4
    for (int c = 0; c < D; ++c) {
      const float kv = rkS[kr * DP + c];
#pragma unroll
      for (int q = 0; q < CH; ++q) acc[q] = route::dot_step(acc[q], rqS[(qb + q) * DP + c], kv);
    }
#pragma unroll
    for (int q = 0; q < CH; ++q) Ts[(qb + q) * KR + kr] = __fmul_rn(acc[q], a.c_d);
    __syncthreads();
    for (int e = tid; e < TI * JC; e += 256) {
      const int r = e / JC, jj = e - r * JC;
      const float* t = Ts + r * KR + jj * W;
      float m = t[0];
      for (int u = 1; u < W; ++u) m = fmaxf(m, t[u]);
      float sum = 0.0f;
      for (int u = 0; u < W; ++u) sum = __fadd_rn(sum, route::rexp_nonpos(__fsub_rn(t[u], m), K));
      const float z = __fadd_rn(__fadd_rn(m, route::rlog(sum, K)), a.bias);
      Gs[r * KR + jj] = __frcp_rn(__fadd_rn(1.0f, route::rexp(-z, K)));
    }
    __syncthreads();
    // compaction: warp w handles rows w, w + 8, ...; lanes over the tile's chunks
    for (int r = warp; r < TI; r += 8) {
      const int i = i0 + r;
      if (i >= a.N) continue;
      const size_t row = ((size_t)bh * a.N + i) * a.N;
      int cnt = cnt_s[r];
      const int j = j0 + lane;
      const bool valid = lane < JC && j < i;
      const float g = lane < JC ? Gs[r * KR + lane] : 0.0f;
      const bool keep = valid && (a.thr <= 0.0f || g >= a.thr);
      const unsigned int bal = __ballot_sync(0xFFFFFFFFu, keep);
      if (keep) {
        const int pos = cnt + __popc(bal & ((1u << lane) - 1u));
        if (a.act_idx) a.act_idx[row + pos] = j;
        if (a.act_g) a.act_g[row + pos] = g;
      }
      if (a.gates_out && lane < JC && j < a.N) a.gates_out[row + j] = valid ? g : 0.0f;
      if (lane == 0) cnt_s[r] = cnt + __popc(bal);
    }
  }
  __syncthreads();
  // counts, zero gates beyond the computed tiles, padding and copies
  for (int r = warp; r < TI; r += 8) {
    const int i = i0 + r;
    if (i >= a.N) continue;
    const size_t row = ((size_t)bh * a.N + i) * a.N;
    const int cnt = cnt_s[r];
    if (lane == 0) {
      if (a.act_cnt) a.act_cnt[(size_t)bh * a.N + i] = cnt;
      if (a.active_cnt_out) a.active_cnt_out[(size_t)bh * a.N + i] = cnt;
    }
    const int jdone = (i_last > 0) ? ((i_last + JC - 1) / JC) * JC : 0;
    if (a.gates_out)
      for (int j = jdone + lane; j < a.N; j += 32) a.gates_out[row + j] = 0.0f;
    if (a.pad_act_idx && a.act_idx)
      for (int p = cnt + lane; p < a.N; p += 32) a.act_idx[row + p] = -1;
    if (a.active_idx_out) {
      __syncwarp();
      for (int p = lane; p < a.N; p += 32) a.active_idx_out[row + p] = p < cnt ? a.act_idx[row + p] : -1;
    }
  }
}

template <int D, int TI>
static cudaError_t launch_gates_window_tiled(const GatesArgs& a, cudaStream_t s) {
  dim3 grid((a.N + TI - 1) / TI, a.B * a.H);
  const size_t smem = (size_t)(TI * (D + 1) + 64 * (D + 1) + 2 * TI * 64 + TI) * 4;
  cudaError_t e = cudaFuncSetAttribute(gates_window_tiled_kernel<D, TI>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  gates_window_tiled_kernel<D, TI><<<grid, 256, smem, s>>>(a);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Launchers
// ---------------------------------------------------------------------------
cudaError_t launch_pools(const void* x0, const void* x1, float* r0, float* r1, int B, int T, int H, int d,
                         int C, int out_chunk_stride, float tau, int dtype, cudaStream_t s) {
  if (C > kPoolMaxC) return cudaErrorInvalidValue;
  const int N = (T + C - 1) / C;
  if (dtype == HLA_BF16 && C <= kTileRows && (H * d) % 64 == 0 && (x0 != nullptr) == (r0 != nullptr) &&
      (x1 != nullptr) == (r1 != nullptr)) {
    PoolTileArgs a{};
    const int nt = (x0 != nullptr) + (x1 != nullptr);
    if (nt == 0) return cudaSuccess;
    // the present tensors first
    a.x[0] = (const __nv_bfloat16*)(x0 ? x0 : x1);
    a.r[0] = x0 ? r0 : r1;
    a.x[1] = (const __nv_bfloat16*)x1;
    a.r[1] = r1;
    a.B = B;
    a.T = T;
    a.H = H;
    a.d = d;
    a.C = C;
    a.N = N;
    a.out_chunk_stride = out_chunk_stride;
    a.groups = H * d / 64;
    a.units = (long)nt * B * N * a.groups;
    a.tau = tau;
    const int smem = kTileWarps * 2 * kTileRows * 128;
    cudaError_t e = cudaFuncSetAttribute(pool_tile_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const long want = (a.units + kTileWarps - 1) / kTileWarps;
    const int blocks = (int)std::min<long>(want, 3L * num_sms());
    pool_tile_kernel<<<blocks, 32 * kTileWarps, smem, s>>>(a);
    return cudaGetLastError();
  }
  const int groups = (H * d + 127) / 128;
  dim3 grid(N, B, 2 * groups);
  if (dtype == HLA_BF16)
    pool_kernel<__nv_bfloat16><<<grid, 64, 0, s>>>((const __nv_bfloat16*)x0, (const __nv_bfloat16*)x1, r0, r1,
                                                     T, H, d, C, out_chunk_stride, tau);
  else
    pool_kernel<float><<<grid, 64, 0, s>>>((const float*)x0, (const float*)x1, r0, r1, T, H, d, C,
                                            out_chunk_stride, tau);
  return cudaGetLastError();
}

cudaError_t launch_gates(const GatesArgs& a, cudaStream_t s) {
  if (a.mode == HLA_GATES_ROUTED && a.win == 0 && (a.d == 128 || a.d == 64)) {
    // 64-row tiles while they give two CTAs per SM or more, else 16-row tiles
    const long tiles64 = (long)((a.N + 63) / 64) * a.B * a.H;
    const bool small = tiles64 < 2L * num_sms();
    if (a.d == 128) return small ? launch_gates_tiled<128, 16>(a, s) : launch_gates_tiled<128, 64>(a, s);
    return small ? launch_gates_tiled<64, 16>(a, s) : launch_gates_tiled<64, 64>(a, s);
  }
  if (a.mode == HLA_GATES_ROUTED && a.win > 0 && 64 % a.win == 0 && (a.d == 128 || a.d == 64)) {
    // 16 query chunks per CTA while that gives two CTAs per SM or more, else 4
    const long tiles16 = (long)((a.N + 15) / 16) * a.B * a.H;
    const bool small = tiles16 < 2L * num_sms();
    if (a.d == 128)
      return small ? launch_gates_window_tiled<128, 4>(a, s) : launch_gates_window_tiled<128, 16>(a, s);
    return small ? launch_gates_window_tiled<64, 4>(a, s) : launch_gates_window_tiled<64, 16>(a, s);
  }
  const long rows = (long)a.B * a.H * a.N;
  const int blocks = (int)((rows * 32 + 255) / 256);
  gates_kernel<<<blocks, 256, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace hla
