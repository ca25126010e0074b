// Intra-chunk read-out on tcgen05 tensor cores, bf16 operands, float32 accumulation.
// d = 128, C = 64.  One CTA (4 warps) per chunk (b, h, i), two CTAs per SM.
//
// HLA summary page, "Methodology in Plain English" para. 3: the current chunk keeps
// weight one and uses its own causal prefix as is, i.e. the token rule runs from
// S_in(i) over chunk i.  With the chunk's WY/UT factors (Wb, Ub, l):
//   O = diag(gamma) Q S_in^T + tril(Gamma o Q K^T) (Ub - Wb S_in^T).
// Two MMAs:
//   MMA1  [Q; Wb] (128 x 128)  x  [S_in; K]^T (128 x 192)  ->  D1 (TMEM, 192 cols):
//         rows 0-63: Q S_in^T | Q K^T;  rows 64-127: Wb S_in^T | (unused)
//   epilogue 1: P = tril(Gamma o Q K^T) (bf16, rows 64-127 zero) and
//               X = Ub - Wb S_in^T (bf16), both into shared memory
//   MMA2  P (128 x 64) x X (64 x 128)  ->  D2 (TMEM)
//   epilogue 2: o_t = gamma_t (Q S_in^T)_t + D2_t, rows t < tokens in the chunk.
// Operands come in by TMA with 128-byte swizzle; P and X reuse the [Q; Wb] buffer.
//
// Channel-wise decay (kChan): with Qt = Q o gamma and Kh = K / gamma per channel
// (chan_prep.cu) the read-out is O = Qt S_in^T + tril(Qt Kh^T) (Ub - Wb S_in^T): the
// same two MMAs with Qt in place of Q and Kh in place of K, no exp in P and no gamma
// row scaling at the end.
#include "common.cuh"
#include "kernels.cuh"
#include "tc_common.cuh"

namespace hla {

HLA_DEFINE_ERROR_WORD(readout_tc)

cudaError_t make_tmap_2d(CUtensorMap* m, const void* base, long inner, long rows, long row_stride_bytes,
                         int box_inner, int box_rows);

namespace {

constexpr int kD = 128;
constexpr int kC = 64;
constexpr int kA1 = 0;                  // [Q; Wb]: 2 K-blocks x 128 rows x 128 B
constexpr int kB1 = 32768;              // [S_in; K]: 2 K-blocks x 192 rows x 128 B
constexpr int kU = kB1 + 2 * 24576;     // Ub: 2 v-halves x 64 rows x 128 B
constexpr int kSmemUsed = kU + 16384;
constexpr int kP = kA1;                 // after MMA1: P (128 rows x 128 B)
constexpr int kX = kA1 + 16384;         // after MMA1: X (2 v-halves x 64 rows x 128 B)
constexpr uint32_t kIdesc1 = tc::idesc_bf16_f32(128, 192, 0, 0);
constexpr uint32_t kIdesc2 = tc::idesc_bf16_f32(128, 128, 0, 1);
constexpr uint32_t kTxBytes = 16384 * 6;  // Q, Wb, S_in (2x), K, Ub

struct ReadoutTcArgs {
  int B, H, T, N;
  const float* ell;  // [B,H,N,C]
  __nv_bfloat16* o;  // [B,T,H,d]
};

__device__ __forceinline__ int swz(int row, int chunk) { return row * 128 + ((chunk ^ (row & 7)) << 4); }

template <bool kChan>
__global__ void __launch_bounds__(128, 2)
    readout_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmU,
                      const __grid_constant__ CUtensorMap tmS, ReadoutTcArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = (uint64_t*)(sm + kSmemUsed);  // tma, mma1, mma2
  uint32_t* tmem_s = (uint32_t*)(bars + 3);
  float* ell_s = (float*)(tmem_s + 4);            // [C]
  volatile int* abort_s = (volatile int*)(ell_s + kC);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int i = blockIdx.x % a.N;
  const int bh = blockIdx.x / a.N;
  const int b = bh / a.H, h = bh % a.H;
  const int t0 = i * kC;
  const int n = min(kC, a.T - t0);
  const long chunk = (long)bh * a.N + i;

  if (tid == 0) {
    for (int k = 0; k < 3; ++k) tc::mbar_init(&bars[k], 1);
    *abort_s = 0;
    tc::mbar_fence_init();
    tc::fence_async_smem();
  }
  if (!kChan && tid < kC) ell_s[tid] = a.ell[chunk * kC + tid];
  if (warp == 0) tc::tmem_alloc(tmem_s, 256);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tm = *tmem_s;

  if (tid == 0) {
    tc::mbar_arrive_expect_tx(&bars[0], kTxBytes);
    const int yq = b * a.T + t0;
    const int yw = (int)(chunk * kC);
    const int ys = (int)(chunk * kD);
    for (int kh = 0; kh < 2; ++kh) {
      // kChan: Qt and Kh are [chunk x 64 rows, 128] like Wb
      tc::tma_load_2d(sm + kA1 + kh * 16384, &tmQ, kChan ? 64 * kh : h * kD + 64 * kh, kChan ? yw : yq, &bars[0]);
      tc::tma_load_2d(sm + kA1 + kh * 16384 + 8192, &tmW, 64 * kh, yw, &bars[0]);
      tc::tma_load_2d(sm + kB1 + kh * 24576, &tmS, 64 * kh, ys, &bars[0]);
      tc::tma_load_2d(sm + kB1 + kh * 24576 + 16384, &tmK, kChan ? 64 * kh : h * kD + 64 * kh, kChan ? yw : yq,
                      &bars[0]);
      tc::tma_load_2d(sm + kU + kh * 8192, &tmU, 64 * kh, yw, &bars[0]);
    }
  }
  bool ok = tc::bar_all(1, 128, tc::mbar_wait(&bars[0], 0, abort_s));
  if (ok && tid == 0) {
    tc::tc_fence_after();
    const uint32_t a_base = tc::smem_u32(sm + kA1), b_base = tc::smem_u32(sm + kB1);
#pragma unroll
    for (int ks = 0; ks < kD / 16; ++ks) {
      const uint64_t ad = tc::sdesc_sw128(a_base + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
      const uint64_t bd = tc::sdesc_sw128(b_base + (ks >> 2) * 24576 + (ks & 3) * 32, 16, 1024);
      tc::mma_ss(tm, ad, bd, kIdesc1, ks > 0 ? 1u : 0u);
    }
    tc::mma_commit(&bars[1]);
  }
  if (ok) ok = tc::bar_all(1, 128, tc::mbar_wait(&bars[1], 0, abort_s));
  if (ok) {
    tc::tc_fence_after();
    const uint32_t lane_addr = tm + ((uint32_t)(32 * warp) << 16);
    const int t = tid;  // row of D1
    if (t < kC) {
      // P row t: Gamma_ts (q_t . k_s) for s <= t
      uint32_t qk[64];
      tc::tmem_ld32(lane_addr + 128, *reinterpret_cast<uint32_t(*)[32]>(&qk[0]));
      tc::tmem_ld32(lane_addr + 160, *reinterpret_cast<uint32_t(*)[32]>(&qk[32]));
      tc::tmem_wait_ld();
      const float lt = kChan ? 0.0f : ell_s[t];
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int s0 = c8 * 8 + 2 * e;
          // kChan: Qt Kh^T is already decayed
          const float d0 = kChan ? 1.0f : __expf(lt - ell_s[s0]);
          const float d1 = kChan ? 1.0f : __expf(lt - ell_s[s0 + 1]);
          const float p0 = s0 <= t ? d0 * __uint_as_float(qk[s0]) : 0.0f;
          const float p1 = s0 + 1 <= t ? d1 * __uint_as_float(qk[s0 + 1]) : 0.0f;
          w[e] = tc::pack_bf16x2(p0, p1);
        }
        *(uint4*)(sm + kP + swz(t, c8)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
    } else {
      // X row s = t - 64: Ub_s - (Wb S_in^T)_s ; P row t is zero
      const int s = t - kC;
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8) *(uint4*)(sm + kP + swz(t, c8)) = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int vh = 0; vh < 2; ++vh) {
        uint32_t ws[64];
        tc::tmem_ld32(lane_addr + 64 * vh, *reinterpret_cast<uint32_t(*)[32]>(&ws[0]));
        tc::tmem_ld32(lane_addr + 64 * vh + 32, *reinterpret_cast<uint32_t(*)[32]>(&ws[32]));
        tc::tmem_wait_ld();
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
          const uint4 u = *(const uint4*)(sm + kU + vh * 8192 + swz(s, c8));
          const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = c8 * 8 + 2 * e;
            w[e] = tc::pack_bf16x2(tc::bf16lo(uw[e]) - __uint_as_float(ws[c]),
                                   tc::bf16hi(uw[e]) - __uint_as_float(ws[c + 1]));
          }
          *(uint4*)(sm + kX + vh * 8192 + swz(s, c8)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
    }
    tc::fence_async_smem();
    tc::tc_fence_before();
  }
  ok = tc::bar_all(1, 128, ok);
  if (ok && tid == 0) {
    tc::tc_fence_after();
    const uint32_t p_base = tc::smem_u32(sm + kP), x_base = tc::smem_u32(sm + kX);
#pragma unroll
    for (int ks = 0; ks < kC / 16; ++ks) {
      const uint64_t ad = tc::sdesc_sw128(p_base + ks * 32, 16, 1024);
      const uint64_t bd = tc::sdesc_sw128(x_base + ks * 2048, 8192, 1024);
      tc::mma_ss(tm + 128, ad, bd, kIdesc2, ks > 0 ? 1u : 0u);
    }
    tc::mma_commit(&bars[2]);
  }
  if (ok) ok = tc::bar_all(1, 128, tc::mbar_wait(&bars[2], 0, abort_s));
  if (ok && tid < kC) {
    tc::tc_fence_after();
    const int t = tid;
    const uint32_t lane_addr = tm + ((uint32_t)(32 * warp) << 16);
    const float gt = kChan ? 1.0f : __expf(ell_s[t]);
    __nv_bfloat16* orow = a.o + (((long)b * a.T + t0 + t) * a.H + h) * kD;
#pragma unroll
    for (int cc = 0; cc < kD; cc += 32) {
      uint32_t y[32], z[32];
      tc::tmem_ld32(lane_addr + cc, y);
      tc::tmem_ld32(lane_addr + 128 + cc, z);
      tc::tmem_wait_ld();
      if (t < n) {
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          w[e] = tc::pack_bf16x2(fmaf(gt, __uint_as_float(y[2 * e]), __uint_as_float(z[2 * e])),
                                 fmaf(gt, __uint_as_float(y[2 * e + 1]), __uint_as_float(z[2 * e + 1])));
        uint4* dst = (uint4*)(orow + cc);
#pragma unroll
        for (int e = 0; e < 4; ++e) dst[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
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

// Readout for bf16, d = 128: q, k [B,T,H,d]; Wb, Ub bf16 [B,H,N,C,d]; S_in bf16
// [B,H,N,d,d] ([v][c]); ell float [B,H,N,C]; o bf16 [B,T,H,d].  With `chan` the
// prepared Qt and Kh ([B,H,N,C,d] bf16) take the places of q and k.
cudaError_t launch_readout_tc(const ReadoutArgs& r, const void* S_in_bf16, const void* Wb_bf16,
                              const void* Ub_bf16, cudaStream_t s, const ChanOperands* chan) {
  if (r.N <= 0) return cudaSuccess;
  const long HD = (long)r.H * kD;
  const long BHN = (long)r.B * r.H * r.N;
  CUtensorMap tq, tk, tw, tu, ts;
  cudaError_t e = cudaSuccess;
  if (chan != nullptr) {
    e = make_tmap_2d(&tq, chan->Qt, kD, BHN * kC, kD * 2, 64, 64);
    if (e == cudaSuccess) e = make_tmap_2d(&tk, chan->Kh, kD, BHN * kC, kD * 2, 64, 64);
  } else {
    e = make_tmap_2d(&tq, r.q, HD, (long)r.B * r.T, HD * 2, 64, 64);
    if (e == cudaSuccess) e = make_tmap_2d(&tk, r.k, HD, (long)r.B * r.T, HD * 2, 64, 64);
  }
  if (e == cudaSuccess) e = make_tmap_2d(&tw, Wb_bf16, kD, BHN * kC, kD * 2, 64, 64);
  if (e == cudaSuccess) e = make_tmap_2d(&tu, Ub_bf16, kD, BHN * kC, kD * 2, 64, 64);
  if (e == cudaSuccess) e = make_tmap_2d(&ts, S_in_bf16, kD, BHN * kD, kD * 2, 64, 128);
  if (e != cudaSuccess) return e;
  ReadoutTcArgs a;
  a.B = r.B;
  a.H = r.H;
  a.T = r.T;
  a.N = r.N;
  a.ell = r.ell;
  a.o = (__nv_bfloat16*)r.o;
  const size_t smem = 1024 + kSmemUsed + 3 * 8 + 16 + kC * 4 + 16;
  if (chan != nullptr) {
    e = cudaFuncSetAttribute(readout_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    readout_tc_kernel<true><<<(unsigned)BHN, 128, smem, s>>>(tq, tk, tw, tu, ts, a);
    return cudaGetLastError();
  }
  e = cudaFuncSetAttribute(readout_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  readout_tc_kernel<false><<<(unsigned)BHN, 128, smem, s>>>(tq, tk, tw, tu, ts, a);
  return cudaGetLastError();
}

}  // namespace hla
