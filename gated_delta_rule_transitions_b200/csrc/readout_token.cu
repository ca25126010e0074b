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
// One CTA per (chunk, head, sequence) with 2 d threads in groups of 8; each thread
// keeps its group's four rows of S on an eighth of the columns (token_rows.cuh): every
// 16-byte shared-memory read of a key, decay or query feeds four rows, the rows
// advance in packed float32 pairs, and a reduce-scatter / all-gather over the group
// forms the per-row dot products.  The keys of the current token stay in registers
// between the dot product and the update.  Keys, queries, decays and values of 16
// tokens at a time are staged in shared memory; the outputs of those tokens are
// gathered there and written row by row.
#include "common.cuh"
#include "kernels.cuh"
#include "token_rows.cuh"

namespace hla {

namespace {

constexpr int kSeg = 16;

template <int D, typename Tio, typename Ts>
__global__ void __launch_bounds__(2 * D, 2) readout_token_kernel(ReadoutTokenArgs a) {
  using namespace token_rows;
  constexpr int E = D / 8;   // columns per thread
  constexpr int M = D / 32;  // 16-byte groups per thread
  constexpr int G = D / 4;   // row groups: rows p, p + G, p + 2G, p + 3G
  __shared__ __align__(16) float ks[kSeg][D];
  __shared__ __align__(16) float qs[kSeg][D];
  __shared__ __align__(16) float as[kSeg][D];
  __shared__ float vs[kSeg][D];
  __shared__ float os[kSeg][D];
  __shared__ float be[kSeg];
  const int i = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int p = threadIdx.x >> 3, g = threadIdx.x & 7;
  const int rown = p + G * owned_row(g);
  const int t0 = i * a.C;
  const int n = min(a.C, a.T - t0);
  const long bh = (long)b * a.H + h;
  const Ts* S = (const Ts*)a.S_in + (bh * a.N + i) * (long)D * D;
  // x01[j] = (rows p, p + G) and x23[j] = (rows p + 2G, p + 3G) at column j
  float2 x01[E], x23[E];
#pragma unroll
  for (int m = 0; m < M; ++m)
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const long c = 32 * m + 4 * g + u;
      x01[4 * m + u] = make_float2(ldf(S + (long)p * D + c), ldf(S + (long)(p + G) * D + c));
      x23[4 * m + u] = make_float2(ldf(S + (long)(p + 2 * G) * D + c), ldf(S + (long)(p + 3 * G) * D + c));
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
      float kr[E];
      float2 d01[2] = {dup(0.0f), dup(0.0f)}, d23[2] = {dup(0.0f), dup(0.0f)};
#pragma unroll
      for (int m = 0; m < M; ++m) {
        const float4 al = a4[8 * m];
        const float4 kk = k4[8 * m];
        const float alv[4] = {al.x, al.y, al.z, al.w};
        kr[4 * m + 0] = kk.x;
        kr[4 * m + 1] = kk.y;
        kr[4 * m + 2] = kk.z;
        kr[4 * m + 3] = kk.w;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int j = 4 * m + u;
          x01[j] = __fmul2_rn(x01[j], dup(alv[u]));
          x23[j] = __fmul2_rn(x23[j], dup(alv[u]));
          d01[u & 1] = __ffma2_rn(x01[j], dup(kr[j]), d01[u & 1]);
          d23[u & 1] = __ffma2_rn(x23[j], dup(kr[j]), d23[u & 1]);
        }
      }
      const float dot = rs_sum4(add2(d01[0], d01[1]), add2(d23[0], d23[1]), g);
      const float bt = be[t];
      float2 f01, f23;
      ag_rows4(bt * dot - bt * vs[t][rown], g, f01, f23);
      const float2 n01 = make_float2(-f01.x, -f01.y), n23 = make_float2(-f23.x, -f23.y);
      float2 y01[2] = {dup(0.0f), dup(0.0f)}, y23[2] = {dup(0.0f), dup(0.0f)};
#pragma unroll
      for (int m = 0; m < M; ++m) {
        const float4 qq = q4[8 * m];
        const float qv[4] = {qq.x, qq.y, qq.z, qq.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int j = 4 * m + u;
          x01[j] = __ffma2_rn(n01, dup(kr[j]), x01[j]);
          x23[j] = __ffma2_rn(n23, dup(kr[j]), x23[j]);
          y01[u & 1] = __ffma2_rn(x01[j], dup(qv[u]), y01[u & 1]);
          y23[u & 1] = __ffma2_rn(x23[j], dup(qv[u]), y23[u & 1]);
        }
      }
      const float y = rs_sum4(add2(y01[0], y01[1]), add2(y23[0], y23[1]), g);
      if ((g & 1) == 0) os[t][rown] = y;
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
