// Intra-chunk read-out by the token rule itself (CUDA cores, float32 arithmetic), for
// channel-wise decay.
//
// HLA summary page, "Methodology in Plain English" para. 3: the current chunk keeps
// weight one and uses its own causal prefix as is, so chunk i runs the token rule
// from its composed state S_in(i) and emits o_t = S_t q_t.  With a decay per key
// channel (the KDA-style decay named in the Gated DeltaNet-2 abstract on the HLA
// listing page) the rule is
//   S_t = S_{t-1} Diag(alpha_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
// and row r of S evolves on its own:
//   s <- s o alpha_t;  s <- s - (beta_t (s . k_t) - beta_t v_t[r]) k_t;  o_t[r] = s . q_t.
// One CTA per (chunk, head, sequence); a pair of threads keeps one row in registers
// (interleaved channels 2j + hf); keys, queries and decays of 16 tokens at a time are
// staged in shared memory.
#include "common.cuh"
#include "kernels.cuh"

namespace hla {

namespace {

constexpr int kSeg = 16;

template <int D, typename Tio, typename Ts>
__global__ void __launch_bounds__(2 * D) readout_token_kernel(ReadoutTokenArgs a) {
  constexpr int E = D / 2;
  __shared__ float ks[kSeg][D];
  __shared__ float qs[kSeg][D];
  __shared__ float as[kSeg][D];
  __shared__ float be[kSeg];
  const int i = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int r = threadIdx.x >> 1, hf = threadIdx.x & 1;
  const int t0 = i * a.C;
  const int n = min(a.C, a.T - t0);
  const long bh = (long)b * a.H + h;
  const Ts* srow = (const Ts*)a.S_in + ((bh * a.N + i) * D + r) * (long)D + hf;
  float x[E];
#pragma unroll
  for (int j = 0; j < E; ++j) x[j] = ldf(srow + 2 * j);
  const long tok0 = b * a.in.sb + h * a.in.sh + (long)t0 * a.in.st;
  const Tio* kin = (const Tio*)a.in.k + tok0;
  const Tio* vin = (const Tio*)a.in.v + tok0;
  const Tio* qin = (const Tio*)a.q + tok0;
  Tio* out = (Tio*)a.o + tok0 + r;
  const long ab0 = b * a.in.ab + h * a.in.ah + (long)t0 * a.in.at;
  for (int s0 = 0; s0 < n; s0 += kSeg) {
    const int ns = min(kSeg, n - s0);
    __syncthreads();
    for (int idx = threadIdx.x; idx < ns * D; idx += 2 * D) {
      const int t = idx / D, cc = idx - t * D;
      ks[t][cc] = ldf(kin + (long)(s0 + t) * a.in.st + cc);
      qs[t][cc] = ldf(qin + (long)(s0 + t) * a.in.st + cc);
      as[t][cc] = a.in.alpha[ab0 + (long)(s0 + t) * a.in.at + cc];
    }
    // the alpha strides are those of beta times d
    if (threadIdx.x < ns) be[threadIdx.x] = a.in.beta[(ab0 + (long)(s0 + threadIdx.x) * a.in.at) / D];
    __syncthreads();
    for (int t = 0; t < ns; ++t) {
#pragma unroll
      for (int j = 0; j < E; ++j) x[j] *= as[t][2 * j + hf];
      float p[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int j = 0; j < E; ++j) p[j & 3] = fmaf(x[j], ks[t][2 * j + hf], p[j & 3]);
      float dot = (p[0] + p[1]) + (p[2] + p[3]);
      dot += __shfl_xor_sync(0xFFFFFFFFu, dot, 1);
      const float bt = be[t];
      const float f = bt * dot - bt * ldf(vin + (long)(s0 + t) * a.in.st + r);
#pragma unroll
      for (int j = 0; j < E; ++j) x[j] = fmaf(-f, ks[t][2 * j + hf], x[j]);
      float o[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int j = 0; j < E; ++j) o[j & 3] = fmaf(x[j], qs[t][2 * j + hf], o[j & 3]);
      float y = (o[0] + o[1]) + (o[2] + o[3]);
      y += __shfl_xor_sync(0xFFFFFFFFu, y, 1);
      if (hf == 0) stf(out + (long)(s0 + t) * a.in.st, y);
    }
  }
}

template <int D, typename Tio>
cudaError_t launch_r(const ReadoutTokenArgs& a, cudaStream_t s) {
  dim3 grid(a.N, a.H, a.B);
  if (a.S_bf16)
    readout_token_kernel<D, Tio, __nv_bfloat16><<<grid, 2 * D, 0, s>>>(a);
  else
    readout_token_kernel<D, Tio, float><<<grid, 2 * D, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_readout_token(const ReadoutTokenArgs& a, cudaStream_t s) {
  if (a.N <= 0) return cudaSuccess;
  if (a.d == 128)
    return a.dtype == HLA_BF16 ? launch_r<128, __nv_bfloat16>(a, s) : launch_r<128, float>(a, s);
  return a.dtype == HLA_BF16 ? launch_r<64, __nv_bfloat16>(a, s) : launch_r<64, float>(a, s);
}

}  // namespace hla
