// Routing kernels: per-chunk log-mean-exp pools, gates and compacted active lists.
// Built with -fmad=false; the recipe itself only uses __f*_rn intrinsics.
#include "common.cuh"
#include "kernels.cuh"
#include "routing_recipe.cuh"

namespace hla {

// ---------------------------------------------------------------------------
// Pools.  grid (N, B, 2), block 256.  blockIdx.z = 0 pools x0 into r0, 1 pools x1
// into r1.  Threads stride over the H*d channels of one chunk; for a fixed token
// the H*d channels are contiguous, so every token row is read coalesced, twice
// (max pass, then sum pass; the second pass hits L2).
// out index: ((b*H + h)*out_chunk_stride + c)*d + ch.
// ---------------------------------------------------------------------------
template <typename Tin>
__global__ void __launch_bounds__(64) pool_kernel(const Tin* __restrict__ x0, const Tin* __restrict__ x1,
                                                  float* __restrict__ r0, float* __restrict__ r1, int T, int H,
                                                  int d, int C, int out_chunk_stride, float tau) {
  // grid (N, B, 2 * groups): blockIdx.z = tensor * groups + group; a group is 128
  // consecutive channels of the H*d channel row; thread = 2 adjacent channels.
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
  const Tin* col = x + ((size_t)b * T + t0) * HD + ch0;
  float m0 = __fmul_rn(ldf(col), inv_tau), m1 = __fmul_rn(ldf(col + 1), inv_tau);
  for (int t = 1; t < n; ++t) {
    m0 = fmaxf(m0, __fmul_rn(ldf(col + (size_t)t * HD), inv_tau));
    m1 = fmaxf(m1, __fmul_rn(ldf(col + (size_t)t * HD + 1), inv_tau));
  }
  float s0 = 0.0f, s1 = 0.0f;
  for (int t = 0; t < n; ++t) {
    s0 = __fadd_rn(s0, route::rexp(__fsub_rn(__fmul_rn(ldf(col + (size_t)t * HD), inv_tau), m0), K));
    s1 = __fadd_rn(s1, route::rexp(__fsub_rn(__fmul_rn(ldf(col + (size_t)t * HD + 1), inv_tau), m1), K));
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
  const float* rk = a.rk + (size_t)bh * a.N * a.d;
  const size_t row = (size_t)warp * a.N;
  int cnt = 0;
  for (int jb = 0; jb < a.N; jb += 32) {
    const int j = jb + lane;
    float g = 0.0f;
    const bool valid = j < i;
    if (valid) {
      if (a.mode == HLA_GATES_ROUTED) {
        const float* rkj = rk + (size_t)j * a.d;
        float dot = 0.0f;
        for (int c = 0; c < a.d; ++c) dot = __fadd_rn(dot, __fmul_rn(rq[c], rkj[c]));
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
// Routed gates, tiled: one CTA per (64 query chunks, b, h).  Each thread computes a
// 4 x 4 block of a 64 x 64 gate tile; every dot product still runs over channels in
// ascending order with separately rounded products and sums, so the bits equal the
// per-pair recipe.  Active chunks are compacted row by row in ascending j.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) gates_tiled_kernel(GatesArgs a) {
  constexpr int TI = 64, TJ = 64;
  extern __shared__ float smf[];
  float(*rqT)[TI] = reinterpret_cast<float(*)[TI]>(smf);            // [D][TI] rq tile, channel-major
  float(*rkT)[TJ] = reinterpret_cast<float(*)[TJ]>(smf + D * TI);   // [D][TJ] rk tile, channel-major
  float(*G)[TJ + 1] = reinterpret_cast<float(*)[TJ + 1]>(smf + 2 * D * TI);  // [TI][TJ+1]
  int* cnt_s = reinterpret_cast<int*>(smf + 2 * D * TI + TI * (TJ + 1));     // [TI]
  const int i0 = blockIdx.x * TI;
  const int bh = blockIdx.y;
  const int tid = threadIdx.x;
  const int ty = tid >> 4, tx = tid & 15;
  const int warp = tid >> 5, lane = tid & 31;
  const route::Consts K = route::make_consts();
  const float* rq = a.rq + (size_t)bh * a.N * D;
  const float* rk = a.rk + (size_t)bh * a.N * D;
  // Tiles are channel-major with their float4 row groups XOR-swizzled by the channel
  // (group g of channel c at slot g ^ (c % 16)): the fill below (one channel, four
  // consecutive rows per thread, one 16-byte store) and the float4 reads of the dot
  // products are both free of bank conflicts.
  for (int e = tid; e < (TI / 4) * D; e += 256) {
    const int g = e / D, c = e - g * D;
    float4 v;
    float* vp = &v.x;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = i0 + 4 * g + u;
      vp[u] = i < a.N ? rq[(size_t)i * D + c] : 0.0f;
    }
    *(float4*)&rqT[c][(g ^ (c & 15)) << 2] = v;
  }
  if (tid < TI) cnt_s[tid] = 0;
  const int i_last = min(a.N, i0 + TI) - 1;
  for (int j0 = 0; j0 < i_last; j0 += TJ) {
    __syncthreads();
    for (int e = tid; e < (TJ / 4) * D; e += 256) {
      const int g = e / D, c = e - g * D;
      float4 v;
      float* vp = &v.x;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int j = j0 + 4 * g + u;
        vp[u] = j < a.N ? rk[(size_t)j * D + c] : 0.0f;
      }
      *(float4*)&rkT[c][(g ^ (c & 15)) << 2] = v;
    }
    __syncthreads();
    float acc[4][4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int w = 0; w < 4; ++w) acc[u][w] = 0.0f;
#pragma unroll 4
    for (int c = 0; c < D; ++c) {
      const float4 q4 = *(const float4*)&rqT[c][(ty ^ (c & 15)) << 2];
      const float4 k4 = *(const float4*)&rkT[c][(tx ^ (c & 15)) << 2];
      const float qv[4] = {q4.x, q4.y, q4.z, q4.w};
      const float kv[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int w = 0; w < 4; ++w) acc[u][w] = __fadd_rn(acc[u][w], __fmul_rn(qv[u], kv[w]));
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int w = 0; w < 4; ++w) G[ty * 4 + u][tx * 4 + w] = route::gate_from_dot(acc[u][w], a.c_d, a.bias, K);
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

// ---------------------------------------------------------------------------
// Launchers
// ---------------------------------------------------------------------------
cudaError_t launch_pools(const void* x0, const void* x1, float* r0, float* r1, int B, int T, int H, int d,
                         int C, int out_chunk_stride, float tau, int dtype, cudaStream_t s) {
  const int N = (T + C - 1) / C;
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
  if (a.mode == HLA_GATES_ROUTED && (a.d == 128 || a.d == 64)) {
    dim3 grid((a.N + 63) / 64, a.B * a.H);
    const size_t smem = (size_t)(2 * a.d * 64 + 64 * 65 + 64) * 4;
    cudaError_t e;
    if (a.d == 128) {
      e = cudaFuncSetAttribute(gates_tiled_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      gates_tiled_kernel<128><<<grid, 256, smem, s>>>(a);
    } else {
      e = cudaFuncSetAttribute(gates_tiled_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      gates_tiled_kernel<64><<<grid, 256, smem, s>>>(a);
    }
    return cudaGetLastError();
  }
  const long rows = (long)a.B * a.H * a.N;
  const int blocks = (int)((rows * 32 + 255) / 256);
  gates_kernel<<<blocks, 256, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace hla
