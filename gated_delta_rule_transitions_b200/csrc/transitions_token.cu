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
#include "token_rows.cuh"

namespace hla {

namespace {

// Tokens staged per step: 32 (keys and values), 16 with channel-wise decay (keys,
// decays and values).
template <bool kChan>
constexpr int seg_len() { return kChan ? 16 : 32; }

// Shared memory (floats): the staged tokens, reused at the end for the output rows
// (d/4 rows at a time).
template <int D, bool kChan>
constexpr int smem_floats() {
  constexpr int stage = seg_len<kChan>() * D * (kChan ? 3 : 2);
  constexpr int outp = (D / 4) * D;
  return stage > outp ? stage : outp;
}

// grid (chunks, H, 2 B): blockIdx.z & 1 selects the rows of A (0) or B (1).  2 d
// threads in groups of 8; each thread keeps its group's four rows on an eighth of the
// columns (token_rows.cuh), so every 16-byte shared-memory read of a key or decay
// feeds four rows, and the keys of the current token stay in registers between the
// dot product and the update.  The rows advance in packed float32 pairs.
// kChan: channel-wise decay, the row is first scaled channel by channel,
//   s <- s o alpha_t,  then  s <- s - (beta_t (s . k_t) - beta_t v_t[r]) k_t.
template <int D, typename Tio, bool kChan>
__global__ void __launch_bounds__(2 * D, 2) transitions_token_kernel(TransArgs a) {
  // a programmatic dependent launched after this grid (the decode close's pool kernel)
  // may be scheduled at once; it waits for this grid before it completes
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  using namespace token_rows;
  constexpr int E = D / 8;   // columns per thread
  constexpr int M = D / 32;  // 16-byte groups per thread
  constexpr int G = D / 4;   // row groups: rows p, p + G, p + 2G, p + 3G
  constexpr int kSeg = seg_len<kChan>();
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
  const int p = threadIdx.x >> 3, g = threadIdx.x & 7;
  const int rown = p + G * owned_row(g);
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
  // x01[j] = (rows p, p + G) and x23[j] = (rows p + 2G, p + 3G) at column j
  float2 x01[E], x23[E];
#pragma unroll
  for (int m = 0; m < M; ++m)
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int cc = 32 * m + 4 * g + u;
      const bool unit = !rowsB && cc % G == p;  // rows of A start at the unit row
      const int q = cc / G;                     // which of the four rows is row cc
      x01[4 * m + u] = make_float2(unit && q == 0 ? 1.0f : 0.0f, unit && q == 1 ? 1.0f : 0.0f);
      x23[4 * m + u] = make_float2(unit && q == 2 ? 1.0f : 0.0f, unit && q == 3 ? 1.0f : 0.0f);
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
      float kr[E];
#pragma unroll
      for (int m = 0; m < M; ++m) {
        const float4 kk = k4[8 * m];
        kr[4 * m + 0] = kk.x;
        kr[4 * m + 1] = kk.y;
        kr[4 * m + 2] = kk.z;
        kr[4 * m + 3] = kk.w;
      }
      if constexpr (kChan) {
        const float4* a4 = (const float4*)&as[t][4 * g];
#pragma unroll
        for (int m = 0; m < M; ++m) {
          const float4 w = a4[8 * m];
          const float wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            x01[4 * m + u] = __fmul2_rn(x01[4 * m + u], dup(wv[u]));
            x23[4 * m + u] = __fmul2_rn(x23[4 * m + u], dup(wv[u]));
          }
        }
      }
      float2 d01[2] = {dup(0.0f), dup(0.0f)}, d23[2] = {dup(0.0f), dup(0.0f)};
#pragma unroll
      for (int j = 0; j < E; ++j) {
        d01[j & 1] = __ffma2_rn(x01[j], dup(kr[j]), d01[j & 1]);
        d23[j & 1] = __ffma2_rn(x23[j], dup(kr[j]), d23[j & 1]);
      }
      const float dot = rs_sum4(add2(d01[0], d01[1]), add2(d23[0], d23[1]), g);
      const float bt = be[t];
      float f;
      if constexpr (kChan)
        f = bt * dot;
      else
        f = al[t] * bt * dot;
      if (rowsB) f -= bt * vs[t][rown];
      float2 f01, f23;
      ag_rows4(f, g, f01, f23);
      const float2 n01 = make_float2(-f01.x, -f01.y), n23 = make_float2(-f23.x, -f23.y);
      if constexpr (kChan) {
#pragma unroll
        for (int j = 0; j < E; ++j) {
          x01[j] = __ffma2_rn(n01, dup(kr[j]), x01[j]);
          x23[j] = __ffma2_rn(n23, dup(kr[j]), x23[j]);
        }
      } else {
        const float2 at2 = dup(al[t]);
#pragma unroll
        for (int j = 0; j < E; ++j) {
          x01[j] = __ffma2_rn(at2, x01[j], __fmul2_rn(n01, dup(kr[j])));
          x23[j] = __ffma2_rn(at2, x23[j], __fmul2_rn(n23, dup(kr[j])));
        }
      }
    }
  }
  // the rows leave through shared memory, a quarter of them at a time, so that the
  // global writes run along rows
  const long bhc = (long)b * a.H + h;
  Tio* out = (Tio*)(rowsB ? a.Bm : a.A) + (bhc * a.ab_chunk_stride + chunk_out + a.ab_chunk_offset) * (long)D * D;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    __syncthreads();
#pragma unroll
    for (int m = 0; m < M; ++m) {
      float w[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float2 v2 = q < 2 ? x01[4 * m + u] : x23[4 * m + u];
        w[u] = (q & 1) ? v2.y : v2.x;
      }
      *(float4*)&sm[p * D + 32 * m + 4 * g] = make_float4(w[0], w[1], w[2], w[3]);
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < G * D; idx += 2 * D) {
      const int rr = idx / D, cc = idx - rr * D;
      stf(out + (long)(q * G + rr) * D + cc, sm[rr * D + cc]);
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
