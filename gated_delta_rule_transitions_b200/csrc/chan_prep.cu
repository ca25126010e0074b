// Channel-wise decay on the tensor cores: the decays of a 64-token sub-chunk folded
// into its keys and queries.
//
// Token rule with a decay per key channel (the KDA-style decay the Gated DeltaNet-2
// abstract on the HLA listing page names; the state's key channels decay each at its
// own rate before the delta-rule edit):
//   S_t = S_{t-1} Diag(alpha_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T.
// With l_t = sum_{s<=t} log alpha_s (a vector over channels) and gamma_t = e^{l_t}, the
// chunkwise WY form keeps the scalar form's shape once the decays sit in the keys:
//   kt_t = k_t o gamma_t,  kh_s = k_s / gamma_s,  kc_s = k_s o gamma_C / gamma_s,
//   qt_t = q_t o gamma_t
//   L  = strictly-lower(diag(beta) Kt Kh^T),  T = (I + L)^{-1} diag(beta)
//   Wb = T Kt,  Ub = T V,  A = Diag(gamma_C) - Wb^T Kc,  B = Ub^T Kc
//   O  = Qt S_in^T + tril(Qt Kh^T) (Ub - Wb S_in^T).
// (kt_t . kh_s = sum_c k_t[c] k_s[c] e^{l_t[c] - l_s[c]}: the decay between the two
// tokens, channel by channel.)  This kernel writes Kt, Kh, Kc and Qt (bf16) and
// gamma_C (float32) for every sub-chunk; the tensor-core transition and read-out
// kernels take them in place of K, Q and their per-token decay scalings.
//
// Range: kh_s = k_s e^{-l_s} grows with the decay accumulated since the sub-chunk's
// first token.  A channel whose decay over one sub-chunk falls below e^{-80} would
// overflow it; the kernel then records kErrDecayRange (hla_device_status reports it)
// and that prefill's outputs are not valid.
//
// One CTA per (sub-chunk, b, h), thread = channel.  Tokens past the end of the
// sequence (a final partial sub-chunk) are identity tokens: alpha = 1, and their
// rows of Kt, Kh, Kc and Qt are zero.
#include "common.cuh"
#include "kernels.cuh"

namespace hla {

HLA_DEFINE_ERROR_WORD(chan_prep)

namespace {

constexpr int kSub = 64;
constexpr int kD = 128;

__global__ void __launch_bounds__(kD) chan_prep_kernel(ChanPrepArgs a) {
  const int sub = blockIdx.x;
  const int bh = blockIdx.y;
  const int b = bh / a.H, h = bh - b * a.H;
  const int c = threadIdx.x;
  const int t0 = sub * kSub;
  const int n = min(kSub, a.T - t0);
  const long HD = (long)a.H * kD;
  const long row0 = ((long)b * a.T + t0) * HD + (long)h * kD + c;  // (b, t0, h, c) of [B,T,H,d]
  // pass 1: l_t per channel (identity tokens past the end: log alpha = 0)
  float ell[kSub];
  float acc = 0.0f;
#pragma unroll
  for (int t = 0; t < kSub; ++t) {
    if (t < n) acc += __logf(a.alpha[row0 + (long)t * HD]);
    ell[t] = acc;
  }
  const long chunk = (long)bh * a.Nsub + sub;
  a.gC[chunk * kD + c] = __expf(acc);
  if (-acc > 80.0f && n > 0) report_device_error(kErrDecayRange);
  // pass 2: the four operands, row t of each at (chunk * 64 + t) * 128 + c
  const __nv_bfloat16* k = (const __nv_bfloat16*)a.k;
  const __nv_bfloat16* q = (const __nv_bfloat16*)a.q;
  __nv_bfloat16* Kt = (__nv_bfloat16*)a.Kt + chunk * kSub * kD + c;
  __nv_bfloat16* Kh = (__nv_bfloat16*)a.Kh + chunk * kSub * kD + c;
  __nv_bfloat16* Kc = (__nv_bfloat16*)a.Kc + chunk * kSub * kD + c;
  __nv_bfloat16* Qt = (__nv_bfloat16*)a.Qt + chunk * kSub * kD + c;
#pragma unroll
  for (int t = 0; t < kSub; ++t) {
    float kv = 0.0f, qv = 0.0f;
    if (t < n) {
      kv = __bfloat162float(k[row0 + (long)t * HD]);
      qv = __bfloat162float(q[row0 + (long)t * HD]);
    }
    const float e = __expf(ell[t]);
    Kt[t * kD] = __float2bfloat16_rn(kv * e);
    Kh[t * kD] = __float2bfloat16_rn(kv * __expf(-ell[t]));
    Kc[t * kD] = __float2bfloat16_rn(kv * __expf(acc - ell[t]));
    Qt[t * kD] = __float2bfloat16_rn(qv * e);
  }
}

}  // namespace

cudaError_t launch_chan_prep(const ChanPrepArgs& a, cudaStream_t s) {
  if (a.Nsub <= 0) return cudaSuccess;
  dim3 grid(a.Nsub, a.B * a.H);
  chan_prep_kernel<<<grid, kD, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace hla
