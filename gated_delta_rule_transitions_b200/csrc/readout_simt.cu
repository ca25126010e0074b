// Intra-chunk read-out on CUDA cores (float32), one CTA per chunk (b, h, i).
//
// HLA summary page, "Methodology in Plain English" para. 3: the current chunk keeps
// weight one and uses its own causal prefix as is, i.e. the token rule runs from
// S_in(i) over chunk i.  In matrix form, with Wb, Ub and l from the chunk's WY/UT
// factors (delta_s = Ub_s - S_in Wb_s is the write of token s):
//   o_t = gamma_t S_in q_t + sum_{s<=t} Gamma_ts (k_s . q_t) (Ub_s - S_in Wb_s)
// i.e.  O = diag(gamma) Q S_in^T + tril(Gamma o Q K^T) (Ub - Wb S_in^T).
#include "common.cuh"
#include "kernels.cuh"

namespace hla {

template <int D, typename Tio>
__global__ void __launch_bounds__(256) readout_simt_kernel(ReadoutArgs a) {
  constexpr int C = 64;
  constexpr int DP = D + 1;
  constexpr int CP = C + 1;
  constexpr int PER = C * D / 256;  // (t, v) outputs per thread
  extern __shared__ float sm[];
  float* Ss = sm;             // [D][DP]  S_in[v][r]
  float* Qs = Ss + D * DP;    // [C][DP]
  float* Ks = Qs + C * DP;    // [C][DP]
  float* Xs = Ks + C * DP;    // [C][DP]  Ub - Wb S_in^T
  float* Ps = Xs + C * DP;    // [C][CP]  tril(Gamma o Q K^T)
  float* ell = Ps + C * CP;   // [C]
  const int i = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x;
  const long bh = (long)b * a.H + h;
  const int t0 = i * C;
  const int n = min(C, a.T - t0);
  const long HD = (long)a.H * D;
  const float* S = a.S_in + (bh * a.N + i) * (long)D * D;
  for (int idx = tid; idx < D * D; idx += blockDim.x) {
    const int v = idx / D, r = idx - v * D;
    Ss[v * DP + r] = S[idx];
  }
  const Tio* qin = (const Tio*)a.q + ((long)b * a.T + t0) * HD + (long)h * D;
  const Tio* kin = (const Tio*)a.k + ((long)b * a.T + t0) * HD + (long)h * D;
  for (int idx = tid; idx < C * D; idx += blockDim.x) {
    const int t = idx / D, c = idx - t * D;
    const bool ok = t < n;
    Qs[t * DP + c] = ok ? ldf(qin + (long)t * HD + c) : 0.0f;
    Ks[t * DP + c] = ok ? ldf(kin + (long)t * HD + c) : 0.0f;
  }
  if (tid < C) ell[tid] = a.ell[(bh * a.N + i) * C + tid];
  __syncthreads();
  const float* Wb = a.Wb + (bh * a.N + i) * (long)C * D;
  const float* Ub = a.Ub + (bh * a.N + i) * (long)C * D;
  float y[PER];
#pragma unroll
  for (int p = 0; p < PER; ++p) {
    const int idx = tid + p * 256;
    const int t = idx / D, v = idx - t * D;
    float yq = 0.0f, yw = 0.0f;
#pragma unroll 8
    for (int r = 0; r < D; ++r) {
      const float s = Ss[v * DP + r];
      yq = fmaf(Qs[t * DP + r], s, yq);
      yw = fmaf(Wb[t * D + r], s, yw);
    }
    y[p] = yq;
    Xs[t * DP + v] = Ub[t * D + v] - yw;
  }
  for (int idx = tid; idx < C * C; idx += blockDim.x) {
    const int t = idx / C, s = idx - t * C;
    float v = 0.0f;
    if (s <= t) {
      float dot = 0.0f;
#pragma unroll 8
      for (int c = 0; c < D; ++c) dot = fmaf(Qs[t * DP + c], Ks[s * DP + c], dot);
      v = expf(ell[t] - ell[s]) * dot;
    }
    Ps[t * CP + s] = v;
  }
  __syncthreads();
  Tio* out = (Tio*)a.o + ((long)b * a.T + t0) * HD + (long)h * D;
#pragma unroll
  for (int p = 0; p < PER; ++p) {
    const int idx = tid + p * 256;
    const int t = idx / D, v = idx - t * D;
    if (t >= n) continue;
    float acc = expf(ell[t]) * y[p];
    for (int s = 0; s <= t; ++s) acc = fmaf(Ps[t * CP + s], Xs[s * DP + v], acc);
    stf(out + (long)t * HD + v, acc);
  }
}

template <int D, typename Tio>
static cudaError_t launch_r(const ReadoutArgs& a, cudaStream_t s) {
  constexpr int C = 64;
  const size_t smem = (size_t)(D * (D + 1) + 3 * C * (D + 1) + C * (C + 1) + C) * sizeof(float);
  auto k = readout_simt_kernel<D, Tio>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.N, a.H, a.B);
  k<<<grid, 256, smem, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_readout(const ReadoutArgs& a, cudaStream_t s) {
  if (a.N <= 0) return cudaSuccess;
  if (a.d == 128)
    return a.dtype == HLA_BF16 ? launch_r<128, __nv_bfloat16>(a, s) : launch_r<128, float>(a, s);
  return a.dtype == HLA_BF16 ? launch_r<64, __nv_bfloat16>(a, s) : launch_r<64, float>(a, s);
}

}  // namespace hla
