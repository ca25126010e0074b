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
__global__ void __launch_bounds__(256) pool_kernel(const Tin* __restrict__ x0, const Tin* __restrict__ x1,
                                                   float* __restrict__ r0, float* __restrict__ r1, int T, int H,
                                                   int d, int C, int out_chunk_stride, float tau) {
  const int c = blockIdx.x;
  const int b = blockIdx.y;
  const Tin* x = blockIdx.z == 0 ? x0 : x1;
  float* r = blockIdx.z == 0 ? r0 : r1;
  if (x == nullptr || r == nullptr) return;
  const route::Consts K = route::make_consts();
  const float inv_tau = __fdiv_rn(1.0f, tau);
  const int t0 = c * C;
  const int n = min(C, T - t0);
  const int HD = H * d;
  for (int ch = threadIdx.x; ch < HD; ch += blockDim.x) {
    const Tin* col = x + ((size_t)b * T + t0) * HD + ch;
    float m = __fmul_rn(ldf(col), inv_tau);
    for (int t = 1; t < n; ++t) m = fmaxf(m, __fmul_rn(ldf(col + (size_t)t * HD), inv_tau));
    float s = 0.0f;
    for (int t = 0; t < n; ++t) {
      const float y = __fmul_rn(ldf(col + (size_t)t * HD), inv_tau);
      s = __fadd_rn(s, route::rexp(__fsub_rn(y, m), K));
    }
    const float mean = __fdiv_rn(s, (float)n);
    const float val = __fmul_rn(tau, __fadd_rn(m, route::rlog(mean, K)));
    const int h = ch / d;
    const int cc = ch - h * d;
    r[(((size_t)b * H + h) * out_chunk_stride + c) * d + cc] = val;
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
// Launchers
// ---------------------------------------------------------------------------
cudaError_t launch_pools(const void* x0, const void* x1, float* r0, float* r1, int B, int T, int H, int d,
                         int C, int out_chunk_stride, float tau, int dtype, cudaStream_t s) {
  const int N = (T + C - 1) / C;
  dim3 grid(N, B, 2);
  if (dtype == HLA_BF16)
    pool_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>((const __nv_bfloat16*)x0, (const __nv_bfloat16*)x1, r0, r1,
                                                     T, H, d, C, out_chunk_stride, tau);
  else
    pool_kernel<float><<<grid, 256, 0, s>>>((const float*)x0, (const float*)x1, r0, r1, T, H, d, C,
                                            out_chunk_stride, tau);
  return cudaGetLastError();
}

cudaError_t launch_gates(const GatesArgs& a, cudaStream_t s) {
  const long rows = (long)a.B * a.H * a.N;
  const int blocks = (int)((rows * 32 + 255) / 256);
  gates_kernel<<<blocks, 256, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace hla
