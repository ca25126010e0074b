// Chunk transitions on CUDA cores (float32 arithmetic), one CTA per (b, h, chunk).
//
// HLA summary page, "Methodology in Plain English" para. 1: affine maps compose, so a
// chunk of tokens is summarised exactly by S -> S A_c + B_c.  The chunkwise WY/UT
// form (named for Gated DeltaNet-2's chunkwise algorithm on the HLA listing page)
// turns the C-fold product of rank-one edits into one triangular solve plus
// products:
//   l_t = sum_{s<=t} log alpha_s, gamma_t = e^{l_t}, Gamma_ts = e^{l_t - l_s}
//   L   = strictly-lower(diag(beta) (Gamma o K K^T))
//   T   = (I + L)^{-1} diag(beta)              (forward substitution)
//   Wb  = T diag(gamma) K,   Ub = T V
//   A_c = gamma_C I - Wb^T D K,  B_c = Ub^T D K,  D = diag(gamma_C / gamma_t)
// The same CTA also writes Wb, Ub and l for the intra-chunk read-out.  A final
// partial chunk is padded with identity tokens (alpha = 1, beta = 0, k = v = 0),
// which change nothing; its A/B are not written.
#include "common.cuh"
#include "kernels.cuh"

namespace hla {

template <int D, typename Tio>
__global__ void __launch_bounds__(256) transitions_simt_kernel(TransArgs a) {
  // a programmatic dependent launched after this grid (the decode close's pool kernel)
  // may be scheduled at once; it waits for this grid before it completes
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  constexpr int C = 64;
  constexpr int DP = D + 1;
  constexpr int CP = C + 1;
  extern __shared__ float sm[];
  float* Ks = sm;               // [C][DP]
  float* Vs = Ks + C * DP;      // [C][DP]
  float* Wb = Vs + C * DP;      // [C][DP]
  float* Ub = Wb + C * DP;      // [C][DP]
  float* Ms = Ub + C * DP;      // [C][CP]  L
  float* Ts = Ms + C * CP;      // [C][CP]  T
  float* al = Ts + C * CP;      // [C]
  float* be = al + C;
  float* ell = be + C;
  float* gam = ell + C;

  const int tid = threadIdx.x;
  const int c = blockIdx.x;
  const int h = blockIdx.y;
  const int b = blockIdx.z;

  long chunk_out = c;
  if (a.close_m != nullptr) {
    // decode close: only sequences whose open chunk becomes full this step
    if (a.close_m[b] + 1 != C) return;
    chunk_out = a.close_n[b];
    if (chunk_out >= a.ab_chunk_stride) return;  // cache full (flagged by the pool kernel)
  }
  const int t0 = c * C;
  const int n = min(C, a.T - t0);
  const bool complete = (n == C);

  const Tio* kin = (const Tio*)a.in.k + b * a.in.sb + h * a.in.sh + (long)t0 * a.in.st;
  const Tio* vin = (const Tio*)a.in.v + b * a.in.sb + h * a.in.sh + (long)t0 * a.in.st;
  for (int idx = tid; idx < C * D; idx += blockDim.x) {
    const int t = idx / D, cc = idx - t * D;
    const bool ok = t < n;
    Ks[t * DP + cc] = ok ? ldf(kin + (long)t * a.in.st + cc) : 0.0f;
    Vs[t * DP + cc] = ok ? ldf(vin + (long)t * a.in.st + cc) : 0.0f;
  }
  if (tid < C) {
    const long off = b * a.in.ab + h * a.in.ah + (long)(t0 + tid) * a.in.at;
    al[tid] = tid < n ? a.in.alpha[off] : 1.0f;
    be[tid] = tid < n ? a.in.beta[off] : 0.0f;
  }
  __syncthreads();
  if (tid == 0) {
    float acc = 0.0f;
    for (int t = 0; t < C; ++t) {
      acc += logf(al[t]);
      ell[t] = acc;
      gam[t] = expf(acc);
    }
  }
  __syncthreads();
  // L = strictly-lower(diag(beta) (Gamma o K K^T))
  for (int idx = tid; idx < C * C; idx += blockDim.x) {
    const int t = idx / C, s = idx - t * C;
    float v = 0.0f;
    if (s < t) {
      float dot = 0.0f;
#pragma unroll 8
      for (int cc = 0; cc < D; ++cc) dot = fmaf(Ks[t * DP + cc], Ks[s * DP + cc], dot);
      v = be[t] * expf(ell[t] - ell[s]) * dot;
    }
    Ms[t * CP + s] = v;
  }
  __syncthreads();
  // T = (I + L)^{-1} diag(beta): column cc by forward substitution
  if (tid < C) {
    const int cc = tid;
    for (int t = 0; t < C; ++t) {
      float acc = 0.0f;
      if (t >= cc) {
        acc = (t == cc) ? be[t] : 0.0f;
        for (int s = cc; s < t; ++s) acc = fmaf(-Ms[t * CP + s], Ts[s * CP + cc], acc);
      }
      Ts[t * CP + cc] = acc;
    }
  }
  __syncthreads();
  // Wb = T diag(gamma) K, Ub = T V
  for (int idx = tid; idx < C * D; idx += blockDim.x) {
    const int t = idx / D, cc = idx - t * D;
    float w = 0.0f, u = 0.0f;
    for (int s = 0; s <= t; ++s) {
      const float tts = Ts[t * CP + s];
      w = fmaf(tts * gam[s], Ks[s * DP + cc], w);
      u = fmaf(tts, Vs[s * DP + cc], u);
    }
    Wb[t * DP + cc] = w;
    Ub[t * DP + cc] = u;
  }
  __syncthreads();
  const long bhc = ((long)b * a.H + h);
  if (a.Wb != nullptr) {
    const long base = (bhc * a.n_chunks + c) * (long)C * D;
    for (int idx = tid; idx < C * D; idx += blockDim.x) {
      const int t = idx / D, cc = idx - t * D;
      a.Wb[base + idx] = Wb[t * DP + cc];
      a.Ub[base + idx] = Ub[t * DP + cc];
    }
    if (tid < C) a.ell[(bhc * a.n_chunks + c) * C + tid] = ell[tid];
  }
  if (complete && a.Kf != nullptr) {
    // factored cache: K, Wb, Ub of the chunk and its scales gamma_C / gamma_t, gamma_C
    const long slot = bhc * a.ab_chunk_stride + chunk_out + a.ab_chunk_offset;
    Tio* Ko = (Tio*)a.Kf + slot * (long)C * D;
    Tio* Wo = (Tio*)a.Wf + slot * (long)C * D;
    Tio* Uo = (Tio*)a.Uf + slot * (long)C * D;
    for (int idx = tid; idx < C * D; idx += blockDim.x) {
      const int t = idx / D, cc = idx - t * D;
      stf(Ko + idx, Ks[t * DP + cc]);
      stf(Wo + idx, Wb[t * DP + cc]);
      stf(Uo + idx, Ub[t * DP + cc]);
    }
    float* dfo = a.df + slot * (long)(C + 4);
    if (tid < C) dfo[tid] = expf(ell[C - 1] - ell[tid]);
    if (tid >= C && tid < C + 4) dfo[tid] = tid == C ? gam[C - 1] : 0.0f;
  }
  if (!complete || a.A == nullptr) return;
  // D K (rows scaled by gamma_C / gamma_t)
  const float lC = ell[C - 1];
  for (int idx = tid; idx < C * D; idx += blockDim.x) {
    const int t = idx / D, cc = idx - t * D;
    Ks[t * DP + cc] *= expf(lC - ell[t]);
  }
  __syncthreads();
  const float gC = gam[C - 1];
  Tio* Aout = (Tio*)a.A + ((bhc * a.ab_chunk_stride) + chunk_out + a.ab_chunk_offset) * (long)D * D;
  Tio* Bout = (Tio*)a.Bm + ((bhc * a.ab_chunk_stride) + chunk_out + a.ab_chunk_offset) * (long)D * D;
  for (int idx = tid; idx < D * D; idx += blockDim.x) {
    const int r = idx / D, cc = idx - r * D;
    float av = 0.0f, bv = 0.0f;
#pragma unroll 8
    for (int t = 0; t < C; ++t) {
      const float dk = Ks[t * DP + cc];
      av = fmaf(Wb[t * DP + r], dk, av);
      bv = fmaf(Ub[t * DP + r], dk, bv);
    }
    stf(Aout + idx, (r == cc ? gC : 0.0f) - av);
    stf(Bout + idx, bv);
  }
}

template <int D, typename Tio>
static cudaError_t launch_t(const TransArgs& a, int chunks, cudaStream_t s) {
  constexpr int C = 64;
  const size_t smem = (size_t)(4 * C * (D + 1) + 2 * C * (C + 1) + 4 * C) * sizeof(float);
  auto k = transitions_simt_kernel<D, Tio>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(chunks, a.H, a.B);
  k<<<grid, 256, smem, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_transitions(const TransArgs& a, cudaStream_t s) {
  const int chunks = a.close_m != nullptr ? 1 : a.n_chunks;
  if (chunks <= 0) return cudaSuccess;
  if (a.d == 128)
    return a.dtype == HLA_BF16 ? launch_t<128, __nv_bfloat16>(a, chunks, s) : launch_t<128, float>(a, chunks, s);
  return a.dtype == HLA_BF16 ? launch_t<64, __nv_bfloat16>(a, chunks, s) : launch_t<64, float>(a, chunks, s);
}

}  // namespace hla
