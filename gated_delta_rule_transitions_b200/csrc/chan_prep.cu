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
// One CTA per (sub-chunk, b, h) of 128 threads: thread = (token half, channel pair),
// so that every access moves two adjacent channels (float2 decays, bf16 pairs).  The
// cumulative sums run in ascending token order (the second half continues from the
// first half's total).  Tokens past the end of the sequence (a final partial
// sub-chunk) are identity tokens: alpha = 1, and their rows of Kt, Kh, Kc and Qt are
// zero.
#include "common.cuh"
#include "kernels.cuh"

namespace hla {

HLA_DEFINE_ERROR_WORD(chan_prep)

namespace {

constexpr int kSub = 64;
constexpr int kHalf = kSub / 2;
constexpr int kD = 128;

__device__ __forceinline__ uint32_t bf16x2_bits(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

__global__ void __launch_bounds__(128) chan_prep_kernel(ChanPrepArgs a) {
  __shared__ float2 tot_s[2][kD / 2];
  const int sub = blockIdx.x;
  const int bh = blockIdx.y;
  const int b = bh / a.H, h = bh - b * a.H;
  const int cp = threadIdx.x & (kD / 2 - 1);  // channels 2 cp, 2 cp + 1
  const int half = threadIdx.x >> 6;          // tokens kHalf * half ...
  const int t0 = sub * kSub;
  const int n = min(kSub, a.T - t0);
  const long HD = (long)a.H * kD;
  const long e0 = ((long)b * a.T + t0) * HD + (long)h * kD + 2 * cp;  // (b, t0, h, 2 cp) of [B,T,H,d]
  // pass 1: log alpha of this thread's tokens (identity tokens past the end: 0) ...
  const float2* alpha2 = reinterpret_cast<const float2*>(a.alpha);
  float2 ell[kHalf];
#pragma unroll
  for (int u = 0; u < kHalf; ++u) {
    const int t = kHalf * half + u;
    ell[u] = make_float2(0.0f, 0.0f);
    if (t < n) {
      const float2 al = alpha2[(e0 + (long)t * HD) >> 1];
      ell[u] = make_float2(__logf(al.x), __logf(al.y));
    }
  }
  // ... then l_t, the running sums over the sub-chunk in ascending t
  float2 acc = make_float2(0.0f, 0.0f);
  if (half == 0) {
#pragma unroll
    for (int u = 0; u < kHalf; ++u) {
      acc.x += ell[u].x;
      acc.y += ell[u].y;
      ell[u] = acc;
    }
    tot_s[0][cp] = acc;
  }
  __syncthreads();
  if (half == 1) {
    acc = tot_s[0][cp];
#pragma unroll
    for (int u = 0; u < kHalf; ++u) {
      acc.x += ell[u].x;
      acc.y += ell[u].y;
      ell[u] = acc;
    }
    tot_s[1][cp] = acc;
  }
  __syncthreads();
  acc = tot_s[1][cp];  // l_C
  const long chunk = (long)bh * a.Nsub + sub;
  if (half == 1) {
    *reinterpret_cast<float2*>(a.gC + chunk * kD + 2 * cp) = make_float2(__expf(acc.x), __expf(acc.y));
    if ((-acc.x > 80.0f || -acc.y > 80.0f) && n > 0) report_device_error(kErrDecayRange);
  }
  // pass 2: the four operands, row t of each at (chunk * 64 + t) * 128 + c
  const uint32_t* k2 = reinterpret_cast<const uint32_t*>(a.k);
  const uint32_t* q2 = reinterpret_cast<const uint32_t*>(a.q);
  const long o0 = (chunk * kSub) * (kD / 2) + cp;  // 32-bit word of (chunk row 0, channel pair cp)
  uint32_t* Kt = reinterpret_cast<uint32_t*>(a.Kt) + o0;
  uint32_t* Kh = reinterpret_cast<uint32_t*>(a.Kh) + o0;
  uint32_t* Kc = reinterpret_cast<uint32_t*>(a.Kc) + o0;
  uint32_t* Qt = reinterpret_cast<uint32_t*>(a.Qt) + o0;
#pragma unroll
  for (int u = 0; u < kHalf; ++u) {
    const int t = kHalf * half + u;
    float k0 = 0.0f, k1 = 0.0f, q0 = 0.0f, q1 = 0.0f;
    if (t < n) {
      const uint32_t kw = k2[(e0 + (long)t * HD) >> 1];
      const uint32_t qw = q2[(e0 + (long)t * HD) >> 1];
      k0 = __uint_as_float(kw << 16);
      k1 = __uint_as_float(kw & 0xFFFF0000u);
      q0 = __uint_as_float(qw << 16);
      q1 = __uint_as_float(qw & 0xFFFF0000u);
    }
    const float ex = __expf(ell[u].x), ey = __expf(ell[u].y);
    const long row = (long)t * (kD / 2);
    Kt[row] = bf16x2_bits(k0 * ex, k1 * ey);
    Kh[row] = bf16x2_bits(k0 * __expf(-ell[u].x), k1 * __expf(-ell[u].y));
    Kc[row] = bf16x2_bits(k0 * __expf(acc.x - ell[u].x), k1 * __expf(acc.y - ell[u].y));
    Qt[row] = bf16x2_bits(q0 * ex, q1 * ey);
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
