// Transitions of chunks longer than 64 tokens by the token rule itself (CUDA cores,
// float32 arithmetic).
//
// HLA summary page, "Methodology in Plain English" para. 1: a chunk acts as the
// affine map S -> S A_c + B_c obtained by applying the per-token rule
//   S <- S alpha_t (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
// over its tokens.  Row by row that is
//   s <- alpha_t s - (alpha_t beta_t (s . k_t) - beta_t v_t[r]) k_t,
// so every row of A_c (started at the unit row e_r, with no write) and of B_c
// (started at zero) evolves on its own.  A pair of threads keeps one row in
// registers; the CTA stages the keys of 64 tokens at a time in shared memory.
//
// Used where no workspace is at hand: the decode step closing a chunk of C > 64
// tokens, and gdn_chunk_transitions at C > 64.  hla_prefill builds the same
// transitions from 64-token WY sub-chunks merged on the tensor cores.
#include "common.cuh"
#include "kernels.cuh"

namespace hla {

namespace {

// Tokens staged per step: 64 (keys only), 32 with channel-wise decay (keys and
// decays), so the static shared memory stays at 32 KiB for d = 128.
template <bool kChan>
constexpr int seg_len() { return kChan ? 32 : 64; }

// grid (chunks, H, 2 B): blockIdx.z & 1 selects the rows of A (0) or B (1).  Two
// threads per row: thread (r, hf) keeps the row's elements 2 j + hf (interleaved, so
// the pair reads adjacent shared-memory words) and the pair adds its dot products.
// kChan: channel-wise decay, the row is first scaled channel by channel,
//   s <- s o alpha_t,  then  s <- s - (beta_t (s . k_t) - beta_t v_t[r]) k_t.
template <int D, typename Tio, bool kChan>
__global__ void __launch_bounds__(2 * D) transitions_token_kernel(TransArgs a) {
  constexpr int E = D / 2;
  constexpr int kSeg = seg_len<kChan>();
  __shared__ float ks[kSeg][D];
  __shared__ float as[kChan ? kSeg : 1][kChan ? D : 1];
  __shared__ float al[kSeg], be[kSeg];
  const int c = blockIdx.x;
  const int h = blockIdx.y;
  const int b = blockIdx.z >> 1;
  const bool rowsB = (blockIdx.z & 1) != 0;
  const int C = a.C;
  const int r = threadIdx.x >> 1;
  const int hf = threadIdx.x & 1;
  long chunk_out = c;
  if (a.close_m != nullptr) {
    // decode close: only sequences whose open chunk becomes full this step
    if (a.close_m[b] + 1 != C) return;
    chunk_out = a.close_n[b];
    if (chunk_out >= a.ab_chunk_stride) return;  // cache full (flagged by the pool kernel)
  }
  const int t0 = c * C;
  if (a.T - t0 < C || a.A == nullptr) return;  // complete chunks only
  const Tio* kin = (const Tio*)a.in.k + b * a.in.sb + h * a.in.sh + (long)t0 * a.in.st;
  const Tio* vin = (const Tio*)a.in.v + b * a.in.sb + h * a.in.sh + (long)t0 * a.in.st;
  const long ab0 = b * a.in.ab + h * a.in.ah + (long)t0 * a.in.at;
  float x[E];
#pragma unroll
  for (int j = 0; j < E; ++j) x[j] = (!rowsB && 2 * j + hf == r) ? 1.0f : 0.0f;
  for (int s0 = 0; s0 < C; s0 += kSeg) {
    __syncthreads();
    for (int idx = threadIdx.x; idx < kSeg * D; idx += 2 * D) {
      const int t = idx / D, cc = idx - t * D;
      ks[t][cc] = ldf(kin + (long)(s0 + t) * a.in.st + cc);
      if constexpr (kChan) as[t][cc] = a.in.alpha[ab0 + (long)(s0 + t) * a.in.at + cc];
    }
    if (threadIdx.x < kSeg) {
      if constexpr (!kChan) al[threadIdx.x] = a.in.alpha[ab0 + (long)(s0 + threadIdx.x) * a.in.at];
      // with channel-wise decay the alpha strides are those of beta times d
      const long bdiv = kChan ? D : 1;
      be[threadIdx.x] = a.in.beta[(ab0 + (long)(s0 + threadIdx.x) * a.in.at) / bdiv];
    }
    __syncthreads();
    for (int t = 0; t < kSeg; ++t) {
      if constexpr (kChan) {
#pragma unroll
        for (int j = 0; j < E; ++j) x[j] *= as[t][2 * j + hf];
      }
      float p[4] = {0.0f, 0.0f, 0.0f, 0.0f};  // four partial sums for latency
#pragma unroll
      for (int j = 0; j < E; ++j) p[j & 3] = fmaf(x[j], ks[t][2 * j + hf], p[j & 3]);
      float dot = (p[0] + p[1]) + (p[2] + p[3]);
      dot += __shfl_xor_sync(0xFFFFFFFFu, dot, 1);
      const float bt = be[t];
      if constexpr (kChan) {
        float f = bt * dot;
        if (rowsB) f -= bt * ldf(vin + (long)(s0 + t) * a.in.st + r);
#pragma unroll
        for (int j = 0; j < E; ++j) x[j] = fmaf(-f, ks[t][2 * j + hf], x[j]);
      } else {
        const float at = al[t];
        float f = at * bt * dot;
        if (rowsB) f -= bt * ldf(vin + (long)(s0 + t) * a.in.st + r);
#pragma unroll
        for (int j = 0; j < E; ++j) x[j] = fmaf(at, x[j], -f * ks[t][2 * j + hf]);
      }
    }
  }
  const long bhc = (long)b * a.H + h;
  Tio* out = (Tio*)(rowsB ? a.Bm : a.A) + (bhc * a.ab_chunk_stride + chunk_out + a.ab_chunk_offset) * (long)D * D +
             (long)r * D + hf;
#pragma unroll
  for (int j = 0; j < E; ++j) stf(out + 2 * j, x[j]);
}

template <int D, typename Tio>
cudaError_t launch_t(const TransArgs& a, int chunks, cudaStream_t s) {
  dim3 grid(chunks, a.H, 2 * a.B);
  if (a.in.alpha_vec)
    transitions_token_kernel<D, Tio, true><<<grid, 2 * D, 0, s>>>(a);
  else
    transitions_token_kernel<D, Tio, false><<<grid, 2 * D, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_transitions_token(const TransArgs& a, cudaStream_t s) {
  if (a.C % 64 != 0) return cudaErrorInvalidValue;
  const int chunks = a.close_m != nullptr ? 1 : a.n_chunks;
  if (chunks <= 0) return cudaSuccess;
  if (a.d == 128)
    return a.dtype == HLA_BF16 ? launch_t<128, __nv_bfloat16>(a, chunks, s) : launch_t<128, float>(a, chunks, s);
  return a.dtype == HLA_BF16 ? launch_t<64, __nv_bfloat16>(a, chunks, s) : launch_t<64, float>(a, chunks, s);
}

}  // namespace hla
