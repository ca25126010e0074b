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
//
// One CTA per (chunk, head, sequence) with 2 d threads.  A thread keeps two rows,
// r0 = p and r1 = p + d/2, restricted to a quarter of the columns, in registers: the
// columns 16 m + 4 g + u (u < 4) for its group index g = thread % 4.  So every
// 16-byte shared-memory read of a key, decay or query is used for both rows, and the
// four threads of a row pair read four adjacent 16-byte words (no bank conflict).
// The two rows advance together in packed float32 pairs (f32x2 arithmetic).  The
// dot products are summed over the four threads by two butterfly shuffles.
// Keys, queries, decays and values of 16 tokens at a time are staged in shared
// memory; the outputs of those tokens are gathered there and written row by row.
#include "common.cuh"
#include "kernels.cuh"

namespace hla {

namespace {

constexpr int kSeg = 16;

template <int D, typename Tio, typename Ts>
__global__ void __launch_bounds__(2 * D, 2) readout_token_kernel(ReadoutTokenArgs a) {
  constexpr int E = D / 4;   // columns per thread and row
  constexpr int M = D / 16;  // 16-byte groups per thread and row
  __shared__ __align__(16) float ks[kSeg][D];
  __shared__ __align__(16) float qs[kSeg][D];
  __shared__ __align__(16) float as[kSeg][D];
  __shared__ float vs[kSeg][D];
  __shared__ float os[kSeg][D];
  __shared__ float be[kSeg];
  const int i = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int p = threadIdx.x >> 2, g = threadIdx.x & 3;
  const int r0 = p, r1 = p + D / 2;
  const int t0 = i * a.C;
  const int n = min(a.C, a.T - t0);
  const long bh = (long)b * a.H + h;
  const Ts* S = (const Ts*)a.S_in + (bh * a.N + i) * (long)D * D;
  // x[j] = (row r0, row r1) at column j: the two rows share every key, decay and
  // query value, so each step is one packed float32 pair operation
  float2 x[E];
#pragma unroll
  for (int m = 0; m < M; ++m)
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int c = 16 * m + 4 * g + u;
      x[4 * m + u] = make_float2(ldf(S + (long)r0 * D + c), ldf(S + (long)r1 * D + c));
    }
  const long tok0 = b * a.in.sb + h * a.in.sh + (long)t0 * a.in.st;
  const Tio* kin = (const Tio*)a.in.k + tok0;
  const Tio* vin = (const Tio*)a.in.v + tok0;
  const Tio* qin = (const Tio*)a.q + tok0;
  Tio* out = (Tio*)a.o + tok0;
  const long ab0 = b * a.in.ab + h * a.in.ah + (long)t0 * a.in.at;
  for (int s0 = 0; s0 < n; s0 += kSeg) {
    const int ns = min(kSeg, n - s0);
    __syncthreads();  // the previous segment's staged inputs and outputs are consumed
    for (int idx = threadIdx.x; idx < ns * D; idx += 2 * D) {
      const int t = idx / D, cc = idx - t * D;
      const long tk = (long)(s0 + t) * a.in.st + cc;
      ks[t][cc] = ldf(kin + tk);
      qs[t][cc] = ldf(qin + tk);
      vs[t][cc] = ldf(vin + tk);
      as[t][cc] = a.in.alpha[ab0 + (long)(s0 + t) * a.in.at + cc];
    }
    // the alpha strides are those of beta times d
    if (threadIdx.x < ns) be[threadIdx.x] = a.in.beta[(ab0 + (long)(s0 + threadIdx.x) * a.in.at) / D];
    __syncthreads();
    for (int t = 0; t < ns; ++t) {
      const float4* a4 = (const float4*)&as[t][4 * g];
      const float4* k4 = (const float4*)&ks[t][4 * g];
      const float4* q4 = (const float4*)&qs[t][4 * g];
      float2 d[2] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)};
#pragma unroll
      for (int m = 0; m < M; ++m) {
        const float4 al = a4[4 * m];
        const float4 kk = k4[4 * m];
        x[4 * m + 0] = __fmul2_rn(x[4 * m + 0], make_float2(al.x, al.x));
        x[4 * m + 1] = __fmul2_rn(x[4 * m + 1], make_float2(al.y, al.y));
        x[4 * m + 2] = __fmul2_rn(x[4 * m + 2], make_float2(al.z, al.z));
        x[4 * m + 3] = __fmul2_rn(x[4 * m + 3], make_float2(al.w, al.w));
        d[m & 1] = __ffma2_rn(x[4 * m + 0], make_float2(kk.x, kk.x), d[m & 1]);
        d[m & 1] = __ffma2_rn(x[4 * m + 1], make_float2(kk.y, kk.y), d[m & 1]);
        d[m & 1] = __ffma2_rn(x[4 * m + 2], make_float2(kk.z, kk.z), d[m & 1]);
        d[m & 1] = __ffma2_rn(x[4 * m + 3], make_float2(kk.w, kk.w), d[m & 1]);
      }
      float dot0 = d[0].x + d[1].x, dot1 = d[0].y + d[1].y;
      dot0 += __shfl_xor_sync(0xFFFFFFFFu, dot0, 1);
      dot1 += __shfl_xor_sync(0xFFFFFFFFu, dot1, 1);
      dot0 += __shfl_xor_sync(0xFFFFFFFFu, dot0, 2);
      dot1 += __shfl_xor_sync(0xFFFFFFFFu, dot1, 2);
      const float bt = be[t];
      const float2 nf = make_float2(-(bt * dot0 - bt * vs[t][r0]), -(bt * dot1 - bt * vs[t][r1]));
      float2 y[2] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)};
#pragma unroll
      for (int m = 0; m < M; ++m) {
        const float4 kk = k4[4 * m];
        const float4 qq = q4[4 * m];
        x[4 * m + 0] = __ffma2_rn(nf, make_float2(kk.x, kk.x), x[4 * m + 0]);
        x[4 * m + 1] = __ffma2_rn(nf, make_float2(kk.y, kk.y), x[4 * m + 1]);
        x[4 * m + 2] = __ffma2_rn(nf, make_float2(kk.z, kk.z), x[4 * m + 2]);
        x[4 * m + 3] = __ffma2_rn(nf, make_float2(kk.w, kk.w), x[4 * m + 3]);
        y[m & 1] = __ffma2_rn(x[4 * m + 0], make_float2(qq.x, qq.x), y[m & 1]);
        y[m & 1] = __ffma2_rn(x[4 * m + 1], make_float2(qq.y, qq.y), y[m & 1]);
        y[m & 1] = __ffma2_rn(x[4 * m + 2], make_float2(qq.z, qq.z), y[m & 1]);
        y[m & 1] = __ffma2_rn(x[4 * m + 3], make_float2(qq.w, qq.w), y[m & 1]);
      }
      float o0 = y[0].x + y[1].x, o1 = y[0].y + y[1].y;
      o0 += __shfl_xor_sync(0xFFFFFFFFu, o0, 1);
      o1 += __shfl_xor_sync(0xFFFFFFFFu, o1, 1);
      o0 += __shfl_xor_sync(0xFFFFFFFFu, o0, 2);
      o1 += __shfl_xor_sync(0xFFFFFFFFu, o1, 2);
      if (g == 0) os[t][r0] = o0;
      if (g == 1) os[t][r1] = o1;
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < ns * D; idx += 2 * D) {
      const int t = idx / D, cc = idx - t * D;
      stf(out + (long)(s0 + t) * a.in.st + cc, os[t][cc]);
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
