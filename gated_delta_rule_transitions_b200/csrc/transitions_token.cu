// Transitions of chunks longer than 64 tokens by the token rule itself (CUDA cores,
// float32 arithmetic).
//
// HLA summary page, "Methodology in Plain English" para. 1: a chunk acts as the
// affine map S -> S A_c + B_c obtained by applying the per-token rule
//   S <- S alpha_t (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
// over its tokens.  Row by row that is
//   s <- alpha_t s - (alpha_t beta_t (s . k_t) - beta_t v_t[r]) k_t,
// so every row of A_c (started at the unit row e_r, with no write) and of B_c
// (started at zero) evolves on its own in registers; the CTA stages the tokens of a
// segment in shared memory.
//
// Used for channel-wise decay (prefill and decode close) and where no workspace is
// at hand: the decode step closing a chunk of C > 64 tokens, and
// gdn_chunk_transitions at C > 64.  With a scalar decay hla_prefill builds the same
// transitions from 64-token WY sub-chunks merged on the tensor cores.
#include "common.cuh"
#include "kernels.cuh"

namespace hla {

namespace {

// Tokens staged per step: 32 (keys and values), 16 with channel-wise decay (keys,
// decays and values).
template <bool kChan>
constexpr int seg_len() { return kChan ? 16 : 32; }

// Shared memory (floats): the staged tokens, reused at the end for the output rows
// (d/2 rows at a time, row stride d + 16 so that the 16-byte stores of the eight
// lanes of one phase fall in distinct banks).
template <int D, bool kChan>
constexpr int smem_floats() {
  constexpr int stage = seg_len<kChan>() * D * (kChan ? 3 : 2);
  constexpr int outp = (D / 2) * (D + 16);
  return stage > outp ? stage : outp;
}

// grid (chunks, H, 2 B): blockIdx.z & 1 selects the rows of A (0) or B (1).  2 d
// threads; a thread keeps rows r0 = p and r1 = p + d/2 restricted to the columns
// 16 m + 4 g + u (u < 4) of its group index g = thread % 4, so every 16-byte
// shared-memory read of a key or decay serves both rows and the four threads of a
// row pair read four adjacent 16-byte words; the two rows advance together in packed
// float32 pairs (f32x2 arithmetic).  Two butterfly shuffles sum the dot products over
// the four threads.
// kChan: channel-wise decay, the row is first scaled channel by channel,
//   s <- s o alpha_t,  then  s <- s - (beta_t (s . k_t) - beta_t v_t[r]) k_t.
template <int D, typename Tio, bool kChan>
__global__ void __launch_bounds__(2 * D, 2) transitions_token_kernel(TransArgs a) {
  constexpr int E = D / 4;   // columns per thread and row
  constexpr int M = D / 16;  // 16-byte groups per thread and row
  constexpr int kSeg = seg_len<kChan>();
  constexpr int kOutStride = D + 16;
  __shared__ __align__(16) float sm[smem_floats<D, kChan>()];
  __shared__ float al[kSeg], be[kSeg];
  float (*ks)[D] = (float (*)[D])sm;
  float (*vs)[D] = (float (*)[D])(sm + kSeg * D);
  float (*as)[D] = (float (*)[D])(sm + 2 * kSeg * D);  // kChan only
  const int c = blockIdx.x;
  const int h = blockIdx.y;
  const int b = blockIdx.z >> 1;
  const bool rowsB = (blockIdx.z & 1) != 0;
  const int C = a.C;
  const int p = threadIdx.x >> 2, g = threadIdx.x & 3;
  const int r0 = p, r1 = p + D / 2;
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
  // x[j] = (row r0, row r1) at column j: one packed float32 pair operation per step
  float2 x[E];
#pragma unroll
  for (int m = 0; m < M; ++m)
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int cc = 16 * m + 4 * g + u;
      x[4 * m + u] = make_float2((!rowsB && cc == r0) ? 1.0f : 0.0f, (!rowsB && cc == r1) ? 1.0f : 0.0f);
    }
  for (int s0 = 0; s0 < C; s0 += kSeg) {
    __syncthreads();
    for (int idx = threadIdx.x; idx < kSeg * D; idx += 2 * D) {
      const int t = idx / D, cc = idx - t * D;
      ks[t][cc] = ldf(kin + (long)(s0 + t) * a.in.st + cc);
      if (rowsB) vs[t][cc] = ldf(vin + (long)(s0 + t) * a.in.st + cc);
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
      const float4* k4 = (const float4*)&ks[t][4 * g];
      if constexpr (kChan) {
        const float4* a4 = (const float4*)&as[t][4 * g];
#pragma unroll
        for (int m = 0; m < M; ++m) {
          const float4 w = a4[4 * m];
          x[4 * m + 0] = __fmul2_rn(x[4 * m + 0], make_float2(w.x, w.x));
          x[4 * m + 1] = __fmul2_rn(x[4 * m + 1], make_float2(w.y, w.y));
          x[4 * m + 2] = __fmul2_rn(x[4 * m + 2], make_float2(w.z, w.z));
          x[4 * m + 3] = __fmul2_rn(x[4 * m + 3], make_float2(w.w, w.w));
        }
      }
      float2 d[2] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)};
#pragma unroll
      for (int m = 0; m < M; ++m) {
        const float4 kk = k4[4 * m];
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
      if constexpr (kChan) {
        float f0 = bt * dot0, f1 = bt * dot1;
        if (rowsB) {
          f0 -= bt * vs[t][r0];
          f1 -= bt * vs[t][r1];
        }
        const float2 nf = make_float2(-f0, -f1);
#pragma unroll
        for (int m = 0; m < M; ++m) {
          const float4 kk = k4[4 * m];
          x[4 * m + 0] = __ffma2_rn(nf, make_float2(kk.x, kk.x), x[4 * m + 0]);
          x[4 * m + 1] = __ffma2_rn(nf, make_float2(kk.y, kk.y), x[4 * m + 1]);
          x[4 * m + 2] = __ffma2_rn(nf, make_float2(kk.z, kk.z), x[4 * m + 2]);
          x[4 * m + 3] = __ffma2_rn(nf, make_float2(kk.w, kk.w), x[4 * m + 3]);
        }
      } else {
        const float at = al[t];
        float f0 = at * bt * dot0, f1 = at * bt * dot1;
        if (rowsB) {
          f0 -= bt * vs[t][r0];
          f1 -= bt * vs[t][r1];
        }
        const float2 nf = make_float2(-f0, -f1), at2 = make_float2(at, at);
#pragma unroll
        for (int m = 0; m < M; ++m) {
          const float4 kk = k4[4 * m];
          x[4 * m + 0] = __ffma2_rn(at2, x[4 * m + 0], __fmul2_rn(nf, make_float2(kk.x, kk.x)));
          x[4 * m + 1] = __ffma2_rn(at2, x[4 * m + 1], __fmul2_rn(nf, make_float2(kk.y, kk.y)));
          x[4 * m + 2] = __ffma2_rn(at2, x[4 * m + 2], __fmul2_rn(nf, make_float2(kk.z, kk.z)));
          x[4 * m + 3] = __ffma2_rn(at2, x[4 * m + 3], __fmul2_rn(nf, make_float2(kk.w, kk.w)));
        }
      }
    }
  }
  // the rows leave through shared memory, half of them at a time, so that the global
  // writes run along rows
  const long bhc = (long)b * a.H + h;
  Tio* out = (Tio*)(rowsB ? a.Bm : a.A) + (bhc * a.ab_chunk_stride + chunk_out + a.ab_chunk_offset) * (long)D * D;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    __syncthreads();
#pragma unroll
    for (int m = 0; m < M; ++m)
      *(float4*)&sm[p * kOutStride + 16 * m + 4 * g] =
          half ? make_float4(x[4 * m + 0].y, x[4 * m + 1].y, x[4 * m + 2].y, x[4 * m + 3].y)
               : make_float4(x[4 * m + 0].x, x[4 * m + 1].x, x[4 * m + 2].x, x[4 * m + 3].x);
    __syncthreads();
    for (int idx = threadIdx.x; idx < (D / 2) * D; idx += 2 * D) {
      const int rr = idx / D, cc = idx - rr * D;
      stf(out + (long)(half * (D / 2) + rr) * D + cc, sm[rr * kOutStride + cc]);
    }
  }
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
