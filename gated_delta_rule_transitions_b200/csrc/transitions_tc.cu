// Chunk transitions on tcgen05 tensor cores: bf16 operands, float32 accumulation and
// float32 triangular solve.  d = 128, C = 64.  One CTA (4 warps) per chunk, two
// CTAs per SM.
//
// HLA summary page, "Methodology in Plain English" para. 1 (a chunk is summarised
// exactly by one affine map S -> S A_c + B_c); chunkwise WY/UT form (the chunkwise WY
// algorithm named in the Gated DeltaNet-2 abstract on the HLA listing page):
//   l_t = sum_{s<=t} log alpha_s, gamma_t = e^{l_t}, Gamma_ts = e^{l_t - l_s}
//   L   = strictly-lower(diag(beta) (Gamma o K K^T)),  T = (I + L)^{-1} diag(beta)
//   Wb  = T diag(gamma) K,  Ub = T V,  D = diag(gamma_C / gamma_t)
//   A_c = gamma_C I - Wb^T D K,  B_c = Ub^T D K.
// MMAs (M is always 128 by stacking):
//   MMA1  [K; V] (128 x 128) x K^T                  -> rows 0-63: K K^T   (64 cols)
//   SIMT  L and the forward substitution for T (float32, shared memory)
//   MMA2  [T diag(gamma); T] (128 x 64) x [K | V]   -> rows 0-63: Wb, rows 64-127: Ub
//   MMA3  Wb^T (128 x 64) x D K (64 x 128)          -> A_c (after gamma_C I - .)
//   MMA4  Ub^T (128 x 64) x D K                     -> B_c
// Wb, Ub (bf16) and l (float32) are also written for the read-out.  A final partial
// chunk (n < C tokens) behaves as if padded with identity tokens (alpha = 1,
// beta = 0): its extra rows of T, Wb and Ub are zero; its A/B are not written.
#include "common.cuh"
#include "kernels.cuh"
#include "tc_common.cuh"

namespace hla {

HLA_DEFINE_ERROR_WORD(transitions_tc)

cudaError_t make_tmap_2d(CUtensorMap* m, const void* base, long inner, long rows, long row_stride_bytes,
                         int box_inner, int box_rows);

namespace {

constexpr int kD = 128;
constexpr int kC = 64;
constexpr int kKV = 0;             // [kh][K | V][64 rows][128 B]   32 KiB
constexpr int kTT = 32768;         // [T gamma; T] 128 rows x 128 B 16 KiB; later D K
constexpr int kScr = 49152;        // L, T float32 [64][65] each; later Wb^T, Ub^T operands
constexpr int kLP = kC + 4;  // row pitch of the float32 L and T (16-byte rows)
constexpr int kSmemUsed = kScr + 2 * kC * kLP * 4;
constexpr uint32_t kIdesc1 = tc::idesc_bf16_f32(128, 64, 0, 0);
constexpr uint32_t kIdesc2 = tc::idesc_bf16_f32(128, 256, 0, 1);
constexpr uint32_t kIdesc3 = tc::idesc_bf16_f32(128, 128, 1, 1);

struct TransTcArgs {
  int B, H, T, N;
  long sb_a, sh_a, st_a;            // alpha/beta strides
  const float* alpha;
  const float* beta;
  __nv_bfloat16* A;                 // [.., chunk_stride, d, d] or null
  __nv_bfloat16* Bm;
  long ab_chunk_stride;
  __nv_bfloat16* Wb;                // [B,H,N,C,d] or null
  __nv_bfloat16* Ub;
  float* ell;                       // [B,H,N,C] or null
};

__device__ __forceinline__ int swz(int row, int chunk) { return row * 128 + ((chunk ^ (row & 7)) << 4); }

__global__ void __launch_bounds__(128, 2)
    transitions_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                          TransTcArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = (uint64_t*)(sm + kSmemUsed);  // tma, m1, m2, m3
  uint32_t* tmem_s = (uint32_t*)(bars + 4);
  float* ell_s = (float*)(tmem_s + 4);           // [C]
  float* beta_s = ell_s + kC;                    // [C]
  float* wsum = beta_s + kC;                     // [2]
  volatile int* abort_s = (volatile int*)(wsum + 2);
  float* Ls = (float*)(sm + kScr);               // [C][kLP]
  float* Ts = Ls + kC * kLP;                     // [C][kLP]

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int i = blockIdx.x % a.N;
  const int bh = blockIdx.x / a.N;
  const int b = bh / a.H, h = bh % a.H;
  const int t0 = i * kC;
  const int n = min(kC, a.T - t0);
  const long chunk = (long)bh * a.N + i;

  if (tid == 0) {
    for (int k = 0; k < 4; ++k) tc::mbar_init(&bars[k], 1);
    *abort_s = 0;
    tc::mbar_fence_init();
    tc::fence_async_smem();
  }
  if (warp == 0) tc::tmem_alloc(tmem_s, 256);
  // l_t = cumulative log alpha (identity tokens beyond n)
  float la = 0.0f;
  if (tid < kC) {
    const long off = b * a.sb_a + h * a.sh_a + (long)(t0 + tid) * a.st_a;
    la = tid < n ? logf(a.alpha[off]) : 0.0f;
    beta_s[tid] = tid < n ? a.beta[off] : 0.0f;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float y = __shfl_up_sync(0xFFFFFFFFu, la, o);
      if (lane >= o) la += y;
    }
    if (lane == 31) wsum[warp] = la;
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tm = *tmem_s;
  if (tid < kC) {
    if (warp == 1) la += wsum[0];
    ell_s[tid] = la;
    if (a.ell) a.ell[chunk * kC + tid] = la;
  }
  if (tid == 0) {
    tc::mbar_arrive_expect_tx(&bars[0], 4 * 8192);
    const int y = b * a.T + t0;
    for (int kh = 0; kh < 2; ++kh) {
      tc::tma_load_2d(sm + kKV + kh * 16384, &tmK, h * kD + 64 * kh, y, &bars[0]);
      tc::tma_load_2d(sm + kKV + kh * 16384 + 8192, &tmV, h * kD + 64 * kh, y, &bars[0]);
    }
  }
  bool ok = tc::bar_all(1, 128, tc::mbar_wait(&bars[0], 0, abort_s));
  // MMA1: [K; V] K^T
  if (ok && tid == 0) {
    tc::tc_fence_after();
    const uint32_t base = tc::smem_u32(sm + kKV);
#pragma unroll
    for (int ks = 0; ks < kD / 16; ++ks) {
      const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
      tc::mma_ss(tm, tc::sdesc_sw128(base + off, 16, 1024), tc::sdesc_sw128(base + off, 16, 1024), kIdesc1,
                 ks > 0 ? 1u : 0u);
    }
    tc::mma_commit(&bars[1]);
  }
  if (ok) ok = tc::bar_all(1, 128, tc::mbar_wait(&bars[1], 0, abort_s));
  const uint32_t lane_addr = tm + ((uint32_t)(32 * warp) << 16);
  if (ok && tid < kC) {
    // L row t
    tc::tc_fence_after();
    const int t = tid;
    uint32_t g[64];
    tc::tmem_ld32(lane_addr, *reinterpret_cast<uint32_t(*)[32]>(&g[0]));
    tc::tmem_ld32(lane_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(&g[32]));
    tc::tmem_wait_ld();
    const float bt = beta_s[t], lt = ell_s[t];
#pragma unroll
    for (int s = 0; s < kC; ++s) Ls[t * kLP + s] = s < t ? bt * __expf(lt - ell_s[s]) * __uint_as_float(g[s]) : 0.0f;
  }
  ok = tc::bar_all(1, 128, ok);
  if (ok && tid < kC) {
    // column c of T = (I + L)^{-1} diag(beta) by forward substitution, fully unrolled
    // so the column stays in registers; every thread runs the same schedule (entries
    // above the diagonal come out as exact zeros), so the reads of L are broadcasts.
    const int c = tid;
    float col[kC];
#pragma unroll
    for (int t = 0; t < kC; ++t) {
      const float* Lrow = Ls + t * kLP;
      float a0 = (t == c) ? beta_s[t] : 0.0f, a1 = 0.0f, a2 = 0.0f, a3 = 0.0f;
#pragma unroll
      for (int s4 = 0; s4 < t; s4 += 4) {
        const float4 l4 = *(const float4*)(Lrow + s4);
        a0 = fmaf(-l4.x, col[s4], a0);
        if (s4 + 1 < t) a1 = fmaf(-l4.y, col[s4 + 1], a1);
        if (s4 + 2 < t) a2 = fmaf(-l4.z, col[s4 + 2], a2);
        if (s4 + 3 < t) a3 = fmaf(-l4.w, col[s4 + 3], a3);
      }
      col[t] = (a0 + a1) + (a2 + a3);
    }
#pragma unroll
    for (int t = 0; t < kC; ++t) Ts[t * kLP + c] = col[t];
  }
  ok = tc::bar_all(1, 128, ok);
  if (ok) {
    // [T diag(gamma); T] as the K-major A operand (rows 0-63 scaled by gamma_s)
    const int t = tid & (kC - 1);
    const bool scaled = tid < kC;
#pragma unroll
    for (int c8 = 0; c8 < 8; ++c8) {
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int s = c8 * 8 + 2 * e;
        float x0 = Ts[t * kLP + s], x1 = Ts[t * kLP + s + 1];
        if (scaled) {
          x0 *= __expf(ell_s[s]);
          x1 *= __expf(ell_s[s + 1]);
        }
        w[e] = tc::pack_bf16x2(x0, x1);
      }
      *(uint4*)(sm + kTT + swz(tid, c8)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    tc::fence_async_smem();
  }
  ok = tc::bar_all(1, 128, ok);
  // MMA2: [T gamma; T] x [K | V]  (N order: K c0-63, V v0-63, K c64-127, V v64-127)
  if (ok && tid == 0) {
    tc::tc_fence_after();
    const uint32_t abase = tc::smem_u32(sm + kTT), bbase = tc::smem_u32(sm + kKV);
#pragma unroll
    for (int ks = 0; ks < kC / 16; ++ks)
      tc::mma_ss(tm, tc::sdesc_sw128(abase + ks * 32, 16, 1024), tc::sdesc_sw128(bbase + ks * 2048, 8192, 1024),
                 kIdesc2, ks > 0 ? 1u : 0u);
    tc::mma_commit(&bars[2]);
  }
  if (ok) ok = tc::bar_all(1, 128, tc::mbar_wait(&bars[2], 0, abort_s));
  if (ok) {
    tc::tc_fence_after();
    // rows 0-63: Wb row t (cols 0-63 and 128-191); rows 64-127: Ub row t (64-127, 192-255)
    const int t = tid & (kC - 1);
    const bool isW = tid < kC;
    uint8_t* opT = sm + kScr + (isW ? 0 : 16384);  // Wb^T / Ub^T operand, [half][64 rows t][128 B]
    __nv_bfloat16* gout = isW ? a.Wb : a.Ub;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      uint32_t x[64];
      const uint32_t col = (isW ? 0 : 64) + 128 * half;
      tc::tmem_ld32(lane_addr + col, *reinterpret_cast<uint32_t(*)[32]>(&x[0]));
      tc::tmem_ld32(lane_addr + col + 32, *reinterpret_cast<uint32_t(*)[32]>(&x[32]));
      tc::tmem_wait_ld();
      uint32_t w[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) w[e] = tc::pack_bf16x2(__uint_as_float(x[2 * e]), __uint_as_float(x[2 * e + 1]));
      if (gout) {
        uint4* dst = (uint4*)(gout + (chunk * kC + t) * kD + 64 * half);
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) dst[c8] = make_uint4(w[4 * c8], w[4 * c8 + 1], w[4 * c8 + 2], w[4 * c8 + 3]);
      }
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8)
        *(uint4*)(opT + half * 8192 + swz(t, c8)) = make_uint4(w[4 * c8], w[4 * c8 + 1], w[4 * c8 + 2], w[4 * c8 + 3]);
    }
    if (isW) {
      // D K row t: K row t scaled by gamma_C / gamma_t, into the old [T gamma; T] space
      const float dt = __expf(ell_s[kC - 1] - ell_s[t]);
#pragma unroll
      for (int half = 0; half < 2; ++half) {
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
          const uint4 kw = *(const uint4*)(sm + kKV + half * 16384 + swz(t, c8));
          const uint32_t kk[4] = {kw.x, kw.y, kw.z, kw.w};
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) w[e] = tc::pack_bf16x2(dt * tc::bf16lo(kk[e]), dt * tc::bf16hi(kk[e]));
          *(uint4*)(sm + kTT + half * 8192 + swz(t, c8)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
    }
    tc::fence_async_smem();
    tc::tc_fence_before();
  }
  ok = tc::bar_all(1, 128, ok);
  const bool write_ab = (n == kC) && a.A != nullptr;
  // MMA3/4: Wb^T D K -> cols 0-127, Ub^T D K -> cols 128-255
  if (ok && write_ab && tid == 0) {
    tc::tc_fence_after();
    const uint32_t wbase = tc::smem_u32(sm + kScr), ubase = wbase + 16384, dbase = tc::smem_u32(sm + kTT);
#pragma unroll
    for (int ks = 0; ks < kC / 16; ++ks) {
      const uint64_t bd = tc::sdesc_sw128(dbase + ks * 2048, 8192, 1024);
      tc::mma_ss(tm, tc::sdesc_sw128(wbase + ks * 2048, 8192, 1024), bd, kIdesc3, ks > 0 ? 1u : 0u);
      tc::mma_ss(tm + 128, tc::sdesc_sw128(ubase + ks * 2048, 8192, 1024), bd, kIdesc3, ks > 0 ? 1u : 0u);
    }
    tc::mma_commit(&bars[3]);
  }
  if (ok && write_ab) ok = tc::bar_all(1, 128, tc::mbar_wait(&bars[3], 0, abort_s));
  if (ok && write_ab) {
    tc::tc_fence_after();
    const int r = tid;
    const float gC = __expf(ell_s[kC - 1]);
    __nv_bfloat16* Arow = a.A + ((long)bh * a.ab_chunk_stride + i) * kD * kD + (long)r * kD;
    __nv_bfloat16* Brow = a.Bm + ((long)bh * a.ab_chunk_stride + i) * kD * kD + (long)r * kD;
#pragma unroll
    for (int cc = 0; cc < kD; cc += 32) {
      uint32_t x[32], y[32];
      tc::tmem_ld32(lane_addr + cc, x);
      tc::tmem_ld32(lane_addr + 128 + cc, y);
      tc::tmem_wait_ld();
      uint32_t wa[16], wb[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int c = cc + 2 * e;
        const float a0 = (r == c ? gC : 0.0f) - __uint_as_float(x[2 * e]);
        const float a1 = (r == c + 1 ? gC : 0.0f) - __uint_as_float(x[2 * e + 1]);
        wa[e] = tc::pack_bf16x2(a0, a1);
        wb[e] = tc::pack_bf16x2(__uint_as_float(y[2 * e]), __uint_as_float(y[2 * e + 1]));
      }
      uint4* da = (uint4*)(Arow + cc);
      uint4* db = (uint4*)(Brow + cc);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        da[e] = make_uint4(wa[4 * e], wa[4 * e + 1], wa[4 * e + 2], wa[4 * e + 3]);
        db[e] = make_uint4(wb[4 * e], wb[4 * e + 1], wb[4 * e + 2], wb[4 * e + 3]);
      }
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (warp == 0) tc::tmem_dealloc(tm, 256);
  if (tid == 0 && *abort_s) report_device_error(kErrMbarTimeout);
}

}  // namespace

// Transitions for bf16, d = 128 over [B,T,H,d] inputs (k, v) and [B,T,H] alpha/beta.
cudaError_t launch_transitions_tc(const TransArgs& t, cudaStream_t s) {
  if (t.n_chunks <= 0) return cudaSuccess;
  const long HD = (long)t.H * kD;
  const long rows = (long)t.B * (t.in.sb / HD);  // B x tokens per sequence
  CUtensorMap tk, tv;
  cudaError_t e = make_tmap_2d(&tk, t.in.k, HD, rows, HD * 2, 64, 64);
  if (e == cudaSuccess) e = make_tmap_2d(&tv, t.in.v, HD, rows, HD * 2, 64, 64);
  if (e != cudaSuccess) return e;
  TransTcArgs a;
  a.B = t.B;
  a.H = t.H;
  a.T = (int)(t.in.sb / HD);  // tokens per sequence in the input layout
  a.N = t.n_chunks;
  a.sb_a = t.in.ab;
  a.sh_a = t.in.ah;
  a.st_a = t.in.at;
  a.alpha = t.in.alpha;
  a.beta = t.in.beta;
  a.A = (__nv_bfloat16*)t.A;
  a.Bm = (__nv_bfloat16*)t.Bm;
  a.ab_chunk_stride = t.ab_chunk_stride;
  a.Wb = (__nv_bfloat16*)t.Wb;
  a.Ub = (__nv_bfloat16*)t.Ub;
  a.ell = t.ell;
  // chunks beyond t.T (gdn_chunk_transitions limits T to whole chunks) are not launched
  const size_t smem = 1024 + kSmemUsed + 4 * 8 + 16 + 2 * kC * 4 + 16;
  e = cudaFuncSetAttribute(transitions_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  transitions_tc_kernel<<<(unsigned)(t.B * t.H * t.n_chunks), 128, smem, s>>>(tk, tv, a);
  return cudaGetLastError();
}

}  // namespace hla
