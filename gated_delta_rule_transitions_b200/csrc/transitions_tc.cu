// Chunk transitions on tcgen05 tensor cores: bf16 operands, float32 accumulation and
// a blocked triangular inverse.  d = 128, C = 64.  Persistent CTAs of 4 warps, two per
// SM, each walking chunks with a grid-wide stride.
//
// HLA summary page, "Methodology in Plain English" para. 1 (a chunk is summarised
// exactly by one affine map S -> S A_c + B_c); chunkwise WY/UT form (the chunkwise WY
// algorithm named in the Gated DeltaNet-2 abstract on the HLA listing page):
//   l_t = sum_{s<=t} log alpha_s, gamma_t = e^{l_t}, Gamma_ts = e^{l_t - l_s}
//   L   = strictly-lower(diag(beta) (Gamma o K K^T)),  T = (I + L)^{-1} diag(beta)
//   Wb  = T diag(gamma) K,  Ub = T V,  D = diag(gamma_C / gamma_t)
//   A_c = gamma_C I - Wb^T D K,  B_c = Ub^T D K.
// Per chunk (M is always 128 by stacking):
//   TMA   K, V tiles (bf16, 128-byte swizzle)
//   MMA1  [K; V] (128 x 128) x K^T                  -> rows 0-63: K K^T   (64 cols)
//   SIMT  L; U = (I + L)^{-1} by 16 x 16 blocks: float32 forward substitution on the
//         four diagonal blocks, then the off-diagonal blocks level by level,
//         U_ij = -sum_{k=j}^{i-1} (U_ii L_ik) U_kj, as warp-level tensor-core products
//         (mma.sync, tf32 inputs, float32 accumulation)
//   MMA2  [T diag(gamma); T] (128 x 64) x [K | V]   -> rows 0-63: Wb, rows 64-127: Ub
//   MMA3  Wb^T (128 x 64) x D K (64 x 128)          -> A_c (after gamma_C I - .)
//   MMA4  Ub^T (128 x 64) x D K                     -> B_c
// Wb, Ub (bf16) and l (float32) are also written for the read-out.  All tile outputs
// leave through TMA stores from swizzled shared memory.  A final partial chunk
// (n < C tokens) behaves as if padded with identity tokens (alpha = 1, beta = 0):
// its extra rows of T, Wb and Ub are zero; its A/B are not written.
//
// Channel-wise decay (kChan): the decays come folded into the keys (chan_prep.cu:
// Kt = K o gamma, Kh = K / gamma, Kc = K o gamma_C / gamma, per channel), so
//   MMA1  [Kt; V] x Kh^T  -> rows 0-63: Kt Kh^T, already decayed (L needs no exp)
//   MMA2  [T; T] x [Kt | V]  (T without a gamma row scaling)
//   MMA3/4 take Kc (loaded by TMA) in place of D K, and A = Diag(gamma_C) - Wb^T Kc.
// Kh is loaded into the T-operand buffer before MMA1, Kc into it after MMA2.
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
constexpr int kKV = 0;                        // [kh][K | V][64 rows][128 B] 32 KiB
constexpr int kTT = 32768;                    // [T gamma; T] 16 KiB; then D K; then B staging (cols 0-63)
constexpr int kScr = 49152;                   // L, U float32; then Wb/Ub operands; then A staging
constexpr int kLP = kC + 4;                   // row pitch (floats) of L and U: 16-byte rows
constexpr int kLU = kC * kLP * 4;             // bytes of one of L, U
constexpr int kX = kScr + 2 * kLU;            // 16 KiB: L' (rows 16-63); then B staging (cols 64-127)
constexpr int kXP = 52;                       // row pitch (floats) of L'
constexpr int kSmall = kX + 16384;            // per-token scalars, barriers
constexpr int kBars = 6;                      // tma, mma1, mma2, mma34, Kh, Kc
constexpr int kSmemUsed = kSmall + 6 * kC * 4 + kBars * 8 + 48;
static_assert(kX % 1024 == 0 && 48 * kXP * 4 <= 16384, "shared-memory layout");
constexpr uint32_t kIdesc1 = tc::idesc_bf16_f32(128, 64, 0, 0);
constexpr uint32_t kIdesc2 = tc::idesc_bf16_f32(128, 256, 0, 1);
constexpr uint32_t kIdesc3 = tc::idesc_bf16_f32(128, 128, 1, 1);

struct TransTcArgs {
  int B, H, T, N;
  long total;                       // B * H * N chunks
  long sb_a, sh_a, st_a;            // alpha strides (scalar decay)
  long sb_b, sh_b, st_b;            // beta strides
  const float* alpha;
  const float* beta;
  bool has_ab;                      // A/B are written (complete chunks)
  long ab_chunk_stride;
  bool has_wu;                      // Wb/Ub are written
  float* ell;                       // [B,H,N,C] or null
  const float* gC;                  // channel-wise decay: gamma_C [total, d]
};

__device__ __forceinline__ int swz(int row, int chunk) { return row * 128 + ((chunk ^ (row & 7)) << 4); }

#ifndef HLA_TRANS_DECAY_PRODUCT
#define HLA_TRANS_DECAY_PRODUCT 1
#endif
// Scalar decay: the pair decays e^{l_t - l_s} of L as e^{l_t} e^{-l_s} (two per-token
// exponentials instead of one per pair) when every |l_t| of the chunk is at most 80,
// so that both factors stay normal float32 numbers; else one exponential per pair.
constexpr bool kDecayProduct = HLA_TRANS_DECAY_PRODUCT != 0;
constexpr float kProductRange = 80.0f;

__device__ __forceinline__ uint32_t to_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}

// d += a b on one 16 x 8 x 8 tile (PTX fragment layout of mma.m16n8k8 with tf32:
// g = lane / 4, q = lane % 4; a: (g, q), (g + 8, q), (g, q + 4), (g + 8, q + 4);
// b: (k = q, n = g), (k = q + 4, n = g); d: (g, 2q), (g, 2q + 1), (g + 8, 2q), (g + 8, 2q + 1)).
__device__ __forceinline__ void mma_tf32_16x8x8(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// acc (16 x 8) = A (16 x KD, row pitch pa floats) times B (KD x 8, row pitch pb), both
// float32 in shared memory; the warp's lanes hold acc in the layout above.
template <int KD>
__device__ __forceinline__ void warp_mma_rows16(float (&acc)[4], const float* A, int pa, const float* B, int pb,
                                                int lane) {
  const int g = lane >> 2, q = lane & 3;
  acc[0] = acc[1] = acc[2] = acc[3] = 0.0f;
#pragma unroll
  for (int k0 = 0; k0 < KD; k0 += 8) {
    const uint32_t af[4] = {to_tf32(A[g * pa + k0 + q]), to_tf32(A[(g + 8) * pa + k0 + q]),
                            to_tf32(A[g * pa + k0 + q + 4]), to_tf32(A[(g + 8) * pa + k0 + q + 4])};
    const uint32_t bf[2] = {to_tf32(B[(k0 + q) * pb + g]), to_tf32(B[(k0 + q + 4) * pb + g])};
    mma_tf32_16x8x8(acc, af, bf);
  }
}

// 32 lanes x 16 columns of 32-bit from tensor memory.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

// Waits for this thread's tensor-memory loads; the registers of the last two loads are
// operands, so no use of them is scheduled before the wait.
__device__ __forceinline__ void tmem_wait_ld_regs(uint32_t (&x)[16], uint32_t (&y)[16]) {
  asm volatile(
      "tcgen05.wait::ld.sync.aligned;"
      : "+r"(x[0]), "+r"(x[1]), "+r"(x[2]), "+r"(x[3]), "+r"(x[4]), "+r"(x[5]), "+r"(x[6]), "+r"(x[7]),
        "+r"(x[8]), "+r"(x[9]), "+r"(x[10]), "+r"(x[11]), "+r"(x[12]), "+r"(x[13]), "+r"(x[14]), "+r"(x[15]),
        "+r"(y[0]), "+r"(y[1]), "+r"(y[2]), "+r"(y[3]), "+r"(y[4]), "+r"(y[5]), "+r"(y[6]), "+r"(y[7]),
        "+r"(y[8]), "+r"(y[9]), "+r"(y[10]), "+r"(y[11]), "+r"(y[12]), "+r"(y[13]), "+r"(y[14]), "+r"(y[15])
      :
      : "memory");
}

__device__ __forceinline__ void tmem_wait_ld_regs(uint32_t (&x)[16]) {
  asm volatile(
      "tcgen05.wait::ld.sync.aligned;"
      : "+r"(x[0]), "+r"(x[1]), "+r"(x[2]), "+r"(x[3]), "+r"(x[4]), "+r"(x[5]), "+r"(x[6]), "+r"(x[7]),
        "+r"(x[8]), "+r"(x[9]), "+r"(x[10]), "+r"(x[11]), "+r"(x[12]), "+r"(x[13]), "+r"(x[14]), "+r"(x[15])
      :
      : "memory");
}

// Stores s * acc at D (16 x 8, row pitch pd).
__device__ __forceinline__ void warp_store_rows16(float* D, int pd, const float (&acc)[4], float s, int lane) {
  const int g = lane >> 2, q = lane & 3;
  *(float2*)(D + g * pd + 2 * q) = make_float2(s * acc[0], s * acc[1]);
  *(float2*)(D + (g + 8) * pd + 2 * q) = make_float2(s * acc[2], s * acc[3]);
}

struct ChunkPos {
  int i, b, h, t0, n;
  long bh;
};

__device__ __forceinline__ ChunkPos chunk_pos(const TransTcArgs& a, long chunk) {
  ChunkPos p;
  p.i = (int)(chunk % a.N);
  p.bh = chunk / a.N;
  p.b = (int)(p.bh / a.H);
  p.h = (int)(p.bh % a.H);
  p.t0 = p.i * kC;
  p.n = min(kC, a.T - p.t0);
  return p;
}

// The position `stride` = qN * N + rN chunks after p (the persistent loop's step),
// without 64-bit divisions: the chunk index wraps into the next (b, h) at most once
// beyond the qN whole heads, and (b, h) is stepped from p's.
__device__ __forceinline__ ChunkPos step_pos(const TransTcArgs& a, const ChunkPos& p, int qN, int rN) {
  ChunkPos n;
  n.i = p.i + rN;
  int dbh = qN;
  if (n.i >= a.N) {
    n.i -= a.N;
    ++dbh;
  }
  n.bh = p.bh + dbh;
  n.h = p.h + dbh;
  n.b = p.b;
  if (n.h >= a.H) {
    const int q = n.h / a.H;
    n.b += q;
    n.h -= q * a.H;
  }
  n.t0 = n.i * kC;
  n.n = min(kC, a.T - n.t0);
  return n;
}

// The K (kChan: Kt, rows chunk * 64 + t of the prepared operand) and V tiles of a chunk.
template <bool kChan>
__device__ __forceinline__ void load_kv(uint8_t* sm, const CUtensorMap* tmK, const CUtensorMap* tmV,
                                        uint64_t* bar, const TransTcArgs& a, const ChunkPos& p, long chunk) {
  tc::mbar_arrive_expect_tx(bar, 4 * 8192);
  const int y = p.b * a.T + p.t0;
  for (int kh = 0; kh < 2; ++kh) {
    if (kChan)
      tc::tma_load_2d(sm + kKV + kh * 16384, tmK, 64 * kh, (int)(chunk * kC), bar);
    else
      tc::tma_load_2d(sm + kKV + kh * 16384, tmK, p.h * kD + 64 * kh, y, bar);
    tc::tma_load_2d(sm + kKV + kh * 16384 + 8192, tmV, p.h * kD + 64 * kh, y, bar);
  }
}

// A 64 x 128 prepared operand (Kh or Kc) of a chunk into the T-operand buffer.
__device__ __forceinline__ void load_tt(uint8_t* sm, const CUtensorMap* tm, uint64_t* bar, long chunk) {
  tc::mbar_arrive_expect_tx(bar, 2 * 8192);
  for (int kh = 0; kh < 2; ++kh) tc::tma_load_2d(sm + kTT + kh * 8192, tm, 64 * kh, (int)(chunk * kC), bar);
}

// alpha, beta of token `tid` of a chunk (identity token beyond n); with a decay per
// channel only beta (the decays are in the prepared operands)
template <bool kChan>
__device__ __forceinline__ void load_ab(const TransTcArgs& a, const ChunkPos& p, int tid, float& al, float& be) {
  if (tid < p.n) {
    al = kChan ? 1.0f : a.alpha[p.b * a.sb_a + p.h * a.sh_a + (long)(p.t0 + tid) * a.st_a];
    be = a.beta[p.b * a.sb_b + p.h * a.sh_b + (long)(p.t0 + tid) * a.st_b];
  } else {
    al = 1.0f;
    be = 0.0f;
  }
}

// Persistent: each CTA walks chunks blockIdx.x, blockIdx.x + gridDim.x, ...; the next
// chunk's K/V tile and alpha/beta are fetched while the current one finishes.
template <bool kChan>
__global__ void __launch_bounds__(128, 2)
    transitions_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                          const __grid_constant__ CUtensorMap tmWb, const __grid_constant__ CUtensorMap tmUb,
                          const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                          const __grid_constant__ CUtensorMap tmKh, const __grid_constant__ CUtensorMap tmKc,
                          TransTcArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  float* Lsm = (float*)(sm + kScr);              // L, [C][kLP]
  float* Usm = (float*)(sm + kScr + kLU);        // U = (I + L)^{-1}, [C][kLP]
  float* Xsm = (float*)(sm + kX);                // L'_ik = U_ii L_ik, rows 16-63, [48][kXP]
  float* ell_s = (float*)(sm + kSmall);          // l_t
  float* beta_s = ell_s + kC;                    // beta_t
  float* bg_s = beta_s + kC;                     // beta_t gamma_t
  float* dk_s = bg_s + kC;                       // gamma_C / gamma_t
  float* gam_s = dk_s + kC;                      // e^{l_t}
  float* igam_s = gam_s + kC;                    // e^{-l_t}
  uint64_t* bars = (uint64_t*)(igam_s + kC);     // tma, mma1, mma2, mma34, Kh, Kc
  uint32_t* tmem_s = (uint32_t*)(bars + kBars);
  float* wsum = (float*)(tmem_s + 2);            // [2]
  uint32_t* lmax_s = (uint32_t*)(wsum + 2);      // [2] largest |l_t| bits of each half chunk
  volatile int* abort_s = (volatile int*)(lmax_s + 2);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  if (tid == 0) {
    for (int k = 0; k < kBars; ++k) tc::mbar_init(&bars[k], 1);
    *abort_s = 0;
    tc::mbar_fence_init();
    tc::fence_async_smem();
  }
  if (warp == 0 && lane == 0) {
    tc::tma_prefetch_desc(&tmK);
    tc::tma_prefetch_desc(&tmV);
    if (a.has_wu) {
      tc::tma_prefetch_desc(&tmWb);
      tc::tma_prefetch_desc(&tmUb);
    }
    if (a.has_ab) {
      tc::tma_prefetch_desc(&tmA);
      tc::tma_prefetch_desc(&tmB);
    }
    if (kChan) {
      tc::tma_prefetch_desc(&tmKh);
      tc::tma_prefetch_desc(&tmKc);
    }
  }
  if (warp == 0) tc::tmem_alloc(tmem_s, 256);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tm = *tmem_s;
  const uint32_t lane_addr = tm + ((uint32_t)(32 * warp) << 16);

  bool ok = true;
  bool load_pending = false;  // thread 0: a K/V load was issued and not yet waited for
  int load_parity = 0;
  int it = 0, ph3 = 0, ph5 = 0;
  bool kh_pending = false, kc_pending = false;  // thread 0 (kChan): a Kh / Kc load in flight
  float pa = 1.0f, pb = 0.0f;  // alpha, beta of token `tid` of the chunk to come
  // this CTA's chunk and the one after it (the loop steps both by gridDim.x)
  const int qN = (int)(gridDim.x / (unsigned)a.N), rN = (int)(gridDim.x % (unsigned)a.N);
  ChunkPos P = chunk_pos(a, blockIdx.x);
  ChunkPos Pn = P;
  if (blockIdx.x < a.total) {
    if (tid == 0) {
      load_kv<kChan>(sm, &tmK, &tmV, &bars[0], a, P, blockIdx.x);
      load_pending = true;
      load_parity = 0;
    }
    if (tid < kC) load_ab<kChan>(a, P, tid, pa, pb);
  }
  for (long chunk = blockIdx.x; ok && chunk < a.total; chunk += gridDim.x, ++it, P = Pn) {
    Pn = step_pos(a, P, qN, rN);  // position of `next`
    const bool write_ab = (P.n == kC) && a.has_ab;
    const long next = chunk + gridDim.x;

    // ---- l_t = cumulative log alpha (a decay per channel: only beta) ----
    float la = 0.0f;
    if (tid < kC) {
      beta_s[tid] = pb;
      if (!kChan) {
        la = logf(pa);
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const float y = __shfl_up_sync(0xFFFFFFFFu, la, o);
          if (lane >= o) la += y;
        }
        if (lane == 31) wsum[warp] = la;
      }
    }
    if (kChan && tid == 0) {
      // Kh into the T-operand buffer, once the previous chunk's staged stores have
      // read it
      tc::bulk_wait_read_all();
      load_tt(sm, &tmKh, &bars[4], chunk);
      kh_pending = true;
    }
    tc::bar_sync(1, 128);
    if (!kChan && tid < kC) {
      if (warp == 1) la += wsum[0];
      ell_s[tid] = la;
      if (a.ell) a.ell[chunk * kC + tid] = la;
      if (kDecayProduct) {
        // |l| >= 0, so its bits order like the values (a NaN compares above every bound)
        const uint32_t m = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(fabsf(la)));
        if (lane == 0) lmax_s[warp] = m;
      }
    }
    // the K/V tile has landed (the previous chunk's staged stores may still be reading
    // shared memory: they are waited for before the L rows are written)
    bool got = true;
    if (tid == 0) {
      got = tc::mbar_wait(&bars[0], it & 1, abort_s);
      if (got) load_pending = false;
      if (kChan && got) {
        got = tc::mbar_wait(&bars[4], it & 1, abort_s);
        if (got) kh_pending = false;
      }
    }
    ok = tc::bar_all(1, 128, got);

    // ---- MMA1: [K; V] K^T -> columns 0-63 (rows 0-63: K K^T; kChan: [Kt; V] Kh^T) ----
    if (ok && tid == 0) {
      tc::tc_fence_after();
      const uint32_t base = tc::smem_u32(sm + kKV);
      const uint32_t bbase = tc::smem_u32(sm + (kChan ? kTT : kKV));
#pragma unroll
      for (int ks = 0; ks < kD / 16; ++ks) {
        const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
        const uint32_t boff = kChan ? (ks >> 2) * 8192 + (ks & 3) * 32 : off;
        tc::mma_ss(tm, tc::sdesc_sw128(base + off, 16, 1024), tc::sdesc_sw128(bbase + boff, 16, 1024), kIdesc1,
                   ks > 0 ? 1u : 0u);
      }
      tc::mma_commit(&bars[1]);
    }
    if (!kChan && ok && tid >= kC) {
      // per-token scales, while the MMA runs
      const int s = tid - kC;
      const float ls = ell_s[s];
      const float e = __expf(ls);
      bg_s[s] = beta_s[s] * e;
      dk_s[s] = __expf(ell_s[kC - 1] - ls);
      if (kDecayProduct) {
        gam_s[s] = e;
        igam_s[s] = __expf(-ls);
      }
    }
    {
      // MMA1 is done and the previous chunk's staged stores have read shared memory
      bool m1 = true;
      if (ok && tid == 0) {
        m1 = tc::mbar_wait(&bars[1], it & 1, abort_s);
        tc::bulk_wait_read_all();
      }
      ok = tc::bar_all(1, 128, ok && m1);
    }

    // ---- L[t][s] = beta_t e^{l_t - l_s} (k_t . k_s) for s < t, else 0 ----
    // warps 0-1 (the lanes of rows 0-63) spill beta_t (K K^T)[t][.]; then every thread
    // applies the decay and the mask to half a row (the exponentials spread over all
    // four sub-partitions)
    if (ok && tid < kC) {
      tc::tc_fence_after();
      const int t = tid;
      uint32_t g[64];
      tc::tmem_ld32(lane_addr, *reinterpret_cast<uint32_t(*)[32]>(&g[0]));
      tc::tmem_ld32(lane_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(&g[32]));
      tc::tmem_wait_ld();
      const float bt = beta_s[t];
      float* Lrow = Lsm + t * kLP;
      if (kChan) {
        // the decays are in Kt Kh^T already: mask the strictly lower part
#pragma unroll
        for (int s4 = 0; s4 < kC; s4 += 4)
          *(float4*)(Lrow + s4) = make_float4(s4 + 0 < t ? bt * __uint_as_float(g[s4 + 0]) : 0.0f,
                                              s4 + 1 < t ? bt * __uint_as_float(g[s4 + 1]) : 0.0f,
                                              s4 + 2 < t ? bt * __uint_as_float(g[s4 + 2]) : 0.0f,
                                              s4 + 3 < t ? bt * __uint_as_float(g[s4 + 3]) : 0.0f);
      } else {
#pragma unroll
        for (int s4 = 0; s4 < kC; s4 += 4)
          *(float4*)(Lrow + s4) = make_float4(bt * __uint_as_float(g[s4]), bt * __uint_as_float(g[s4 + 1]),
                                              bt * __uint_as_float(g[s4 + 2]), bt * __uint_as_float(g[s4 + 3]));
      }
      tc::tc_fence_before();
    }
    ok = tc::bar_all(1, 128, ok);
    const bool product = kDecayProduct && max(lmax_s[0], lmax_s[1]) <= __float_as_uint(kProductRange);
    if (!kChan && ok && product) {
      const int t = tid & (kC - 1), hs = tid >> 6;
      const float gt = gam_s[t];
      float* Lrow = Lsm + t * kLP;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int s4 = 32 * hs + 4 * q;
        const float4 i4 = *(const float4*)(igam_s + s4);
        const float4 g4 = *(const float4*)(Lrow + s4);
        float4 v;
        v.x = (s4 + 0 < t) ? (gt * i4.x) * g4.x : 0.0f;
        v.y = (s4 + 1 < t) ? (gt * i4.y) * g4.y : 0.0f;
        v.z = (s4 + 2 < t) ? (gt * i4.z) * g4.z : 0.0f;
        v.w = (s4 + 3 < t) ? (gt * i4.w) * g4.w : 0.0f;
        *(float4*)(Lrow + s4) = v;
      }
    } else if (!kChan && ok) {
      const int t = tid & (kC - 1), hs = tid >> 6;
      const float lt = ell_s[t];
      float* Lrow = Lsm + t * kLP;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int s4 = 32 * hs + 4 * q;
        const float4 l4 = *(const float4*)(ell_s + s4);
        const float4 g4 = *(const float4*)(Lrow + s4);
        float4 v;
        v.x = (s4 + 0 < t) ? __expf(lt - l4.x) * g4.x : 0.0f;
        v.y = (s4 + 1 < t) ? __expf(lt - l4.y) * g4.y : 0.0f;
        v.z = (s4 + 2 < t) ? __expf(lt - l4.z) * g4.z : 0.0f;
        v.w = (s4 + 3 < t) ? __expf(lt - l4.w) * g4.w : 0.0f;
        *(float4*)(Lrow + s4) = v;
      }
    }
    ok = tc::bar_all(1, 128, ok);

    // ---- U = (I + L)^{-1} by 16 x 16 blocks.  Diagonal blocks U_kk: forward
    //      substitution, thread = (block k, column c) ----
    if (ok && tid < kC) {
      const int k = tid >> 4, c = tid & 15;
      float x[16];
#pragma unroll
      for (int tl = 0; tl < 16; ++tl) {
        const float* Lrow = Lsm + (16 * k + tl) * kLP + 16 * k;
        float v = (tl == c) ? 1.0f : 0.0f;
#pragma unroll
        for (int sl = 0; sl < tl; ++sl) v = fmaf(-Lrow[sl], x[sl], v);
        x[tl] = v;
      }
#pragma unroll
      for (int tl = 0; tl < 16; ++tl) Usm[(16 * k + tl) * kLP + 16 * k + c] = x[tl];
    }
    ok = tc::bar_all(1, 128, ok);
    // Off-diagonal blocks.  With L'_ik = U_ii L_ik (k < i),  U_ij = -sum_{k=j}^{i-1} L'_ik U_kj,
    // one level (i - j = 1, 2, 3) after the other.
    {
      // warp-level products (tf32 inputs, float32 accumulation): a unit is one 16 x 8
      // half (column half nh) of a block
      if (ok) {
        // L'_ik for (i, k) = (1,0) (2,0) (2,1) (3,0) (3,1) (3,2): 12 units, 3 per warp
#pragma unroll
        for (int r = 0; r < 3; ++r) {
          const int u = warp + 4 * r, blk = u >> 1, nh = u & 1;
          const int ib = blk < 1 ? 1 : (blk < 3 ? 2 : 3);
          const int kb = blk - (ib * (ib - 1)) / 2;
          float acc[4];
          warp_mma_rows16<16>(acc, Usm + 16 * ib * kLP + 16 * ib, kLP, Lsm + 16 * ib * kLP + 16 * kb + 8 * nh, kLP,
                              lane);
          warp_store_rows16(Xsm + (16 * ib - 16) * kXP + 16 * kb + 8 * nh, kXP, acc, 1.0f, lane);
        }
      }
      ok = tc::bar_all(1, 128, ok);
      if (ok) {
        // level 1: U_{j+1,j} = -L'_{j+1,j} U_jj, j = 0, 1, 2 (6 units)
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int u = warp + 4 * r;
          if (u < 6) {
            const int jb = u >> 1, nh = u & 1;
            float acc[4];
            warp_mma_rows16<16>(acc, Xsm + 16 * jb * kXP + 16 * jb, kXP, Usm + 16 * jb * kLP + 16 * jb + 8 * nh, kLP,
                                lane);
            warp_store_rows16(Usm + 16 * (jb + 1) * kLP + 16 * jb + 8 * nh, kLP, acc, -1.0f, lane);
          }
        }
      }
      ok = tc::bar_all(1, 128, ok);
      if (ok) {
        // level 2: U_{j+2,j} = -(L'_{j+2,j} U_jj + L'_{j+2,j+1} U_{j+1,j}), j = 0, 1 (4 units)
        const int jb = warp >> 1, nh = warp & 1;
        float acc[4];
        warp_mma_rows16<32>(acc, Xsm + 16 * (jb + 1) * kXP + 16 * jb, kXP, Usm + 16 * jb * kLP + 16 * jb + 8 * nh,
                            kLP, lane);
        warp_store_rows16(Usm + 16 * (jb + 2) * kLP + 16 * jb + 8 * nh, kLP, acc, -1.0f, lane);
      }
      ok = tc::bar_all(1, 128, ok);
      if (ok && warp < 2) {
        // level 3: U_30 = -(L'_30 U_00 + L'_31 U_10 + L'_32 U_20) (2 units)
        float acc[4];
        warp_mma_rows16<48>(acc, Xsm + 32 * kXP, kXP, Usm + 8 * warp, kLP, lane);
        warp_store_rows16(Usm + 48 * kLP + 8 * warp, kLP, acc, -1.0f, lane);
      }
      ok = tc::bar_all(1, 128, ok);
    }

    // ---- operand [T diag(gamma); T] (bf16, K-major, 128 rows x 64), T = U diag(beta) ----
    if (ok) {
      const int r = tid, t = r & (kC - 1);
      const float* scl = (!kChan && r < kC) ? bg_s : beta_s;
      const float* Urow = Usm + t * kLP;
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8) {
        uint4 w = make_uint4(0u, 0u, 0u, 0u);
        if ((c8 >> 1) <= (t >> 4)) {  // blocks above the diagonal are zero
          const float4 u0 = *(const float4*)(Urow + 8 * c8);
          const float4 u1 = *(const float4*)(Urow + 8 * c8 + 4);
          const float4 s0 = *(const float4*)(scl + 8 * c8);
          const float4 s1 = *(const float4*)(scl + 8 * c8 + 4);
          w.x = tc::pack_bf16x2(u0.x * s0.x, u0.y * s0.y);
          w.y = tc::pack_bf16x2(u0.z * s0.z, u0.w * s0.w);
          w.z = tc::pack_bf16x2(u1.x * s1.x, u1.y * s1.y);
          w.w = tc::pack_bf16x2(u1.z * s1.z, u1.w * s1.w);
        }
        *(uint4*)(sm + kTT + swz(r, c8)) = w;
      }
      tc::fence_async_smem();
    }
    ok = tc::bar_all(1, 128, ok);

    // ---- MMA2: [T gamma; T] x [K | V]  (N order: K c0-63, V v0-63, K c64-127, V v64-127) ----
    if (ok && tid == 0) {
      tc::tc_fence_after();
      const uint32_t abase = tc::smem_u32(sm + kTT), bbase = tc::smem_u32(sm + kKV);
#pragma unroll
      for (int ks = 0; ks < kC / 16; ++ks)
        tc::mma_ss(tm, tc::sdesc_sw128(abase + ks * 32, 16, 1024), tc::sdesc_sw128(bbase + ks * 2048, 8192, 1024),
                   kIdesc2, ks > 0 ? 1u : 0u);
      tc::mma_commit(&bars[2]);
    }
    {
      const bool m2 = (ok && tid == 0) ? tc::mbar_wait(&bars[2], it & 1, abort_s) : true;
      // kChan: the T operand has been read; Kc takes its buffer for MMA3/4
      if (kChan && ok && m2 && tid == 0 && write_ab) {
        load_tt(sm, &tmKc, &bars[5], chunk);
        kc_pending = true;
      }
      ok = tc::bar_all(1, 128, ok && m2);
    }

    // ---- Wb (rows 0-63) and Ub (rows 64-127) to bf16 row-major swizzled tiles in Scr:
    //      the MN-major A operands of MMA3/4 and the sources of their TMA stores;
    //      D K (K row t scaled by gamma_C / gamma_t) into TT ----
    if (ok) {
      tc::tc_fence_after();
      const int t = tid & (kC - 1);
      const bool isW = tid < kC;
      uint8_t* opT = sm + kScr + (isW ? 0 : 16384);  // [half][64 rows t][128 B]
      // the row's 128 columns (K half 0: 0-63, half 1: 128-191; V at +64) in pieces of 16;
      // the next piece's tensor-memory load is in flight while one is converted and
      // stored, and the first one while D K is built
      const uint32_t col0 = isW ? 0 : 64;
      uint32_t x[2][16];
      tmem_ld16(lane_addr + col0, x[0]);
      if (!kChan) {
        // D K: row t, columns 64 half .. 64 half + 63 (warps 0-1 the first half, 2-3 the second)
        const float dt = dk_s[t];
        const int half = tid >> 6;
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
      tmem_wait_ld_regs(x[0]);
#pragma unroll
      for (int pc = 0; pc < 8; ++pc) {
        const int cur = pc & 1;
        if (pc + 1 < 8)
          tmem_ld16(lane_addr + col0 + 128 * ((pc + 1) >> 2) + 16 * ((pc + 1) & 3), x[cur ^ 1]);
        const int half = pc >> 2;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int c8 = 2 * (pc & 3) + c;
          uint4 w;
          w.x = tc::pack_bf16x2(__uint_as_float(x[cur][8 * c + 0]), __uint_as_float(x[cur][8 * c + 1]));
          w.y = tc::pack_bf16x2(__uint_as_float(x[cur][8 * c + 2]), __uint_as_float(x[cur][8 * c + 3]));
          w.z = tc::pack_bf16x2(__uint_as_float(x[cur][8 * c + 4]), __uint_as_float(x[cur][8 * c + 5]));
          w.w = tc::pack_bf16x2(__uint_as_float(x[cur][8 * c + 6]), __uint_as_float(x[cur][8 * c + 7]));
          *(uint4*)(opT + half * 8192 + swz(t, c8)) = w;
        }
        if (pc + 1 < 8) tmem_wait_ld_regs(x[cur ^ 1]);
      }
      tc::fence_async_smem();
      tc::tc_fence_before();
    }
    ok = tc::bar_all(1, 128, ok);
    const bool mma34 = ok && write_ab;
    if (ok && tid == 0) {
      tc::tc_fence_after();
      // kChan: Kc has landed in the T-operand buffer
      bool kc_ok = true;
      if (kChan && kc_pending) {
        kc_ok = tc::mbar_wait(&bars[5], ph5 & 1, abort_s);
        if (kc_ok) {
          kc_pending = false;
          ++ph5;
        }
      }
      // MMA3/4: Wb^T D K -> columns 0-127, Ub^T D K -> columns 128-255 (kChan: Kc for D K)
      if (mma34 && kc_ok) {
        const uint32_t wbase = tc::smem_u32(sm + kScr), ubase = wbase + 16384, dbase = tc::smem_u32(sm + kTT);
#pragma unroll
        for (int ks = 0; ks < kC / 16; ++ks) {
          const uint64_t bd = tc::sdesc_sw128(dbase + ks * 2048, 8192, 1024);
          tc::mma_ss(tm, tc::sdesc_sw128(wbase + ks * 2048, 8192, 1024), bd, kIdesc3, ks > 0 ? 1u : 0u);
          tc::mma_ss(tm + 128, tc::sdesc_sw128(ubase + ks * 2048, 8192, 1024), bd, kIdesc3, ks > 0 ? 1u : 0u);
        }
        tc::mma_commit(&bars[3]);
      }
      // Wb/Ub leave from the same tiles MMA3/4 read (both only read them)
      if (a.has_wu) {
        const int y = (int)(chunk * kC);
        tc::tma_store_2d(&tmWb, sm + kScr, 0, y);
        tc::tma_store_2d(&tmWb, sm + kScr + 8192, 64, y);
        tc::tma_store_2d(&tmUb, sm + kScr + 16384, 0, y);
        tc::tma_store_2d(&tmUb, sm + kScr + 16384 + 8192, 64, y);
        tc::bulk_commit();
      }
      // the K/V tile is no longer read (MMA2 done, D K built): fetch the next chunk's
      if (next < a.total) {
        load_kv<kChan>(sm, &tmK, &tmV, &bars[0], a, Pn, next);
        load_pending = true;
        load_parity = (it + 1) & 1;
      }
    }
    if (ok && tid < kC && next < a.total) load_ab<kChan>(a, Pn, tid, pa, pb);
    if (mma34) {
      const bool m3 = tid == 0 ? tc::mbar_wait(&bars[3], ph3 & 1, abort_s) : true;
      ++ph3;
      if (tid == 0 && m3) tc::bulk_wait_read_all();  // the Wb/Ub stores have read Scr
      ok = tc::bar_all(1, 128, m3);
    }

    // ---- A = gamma_C I - Wb^T D K and B = Ub^T D K (row r per thread) to bf16 swizzled
    //      staging (A in Scr; B in TT and X), then TMA stores ----
    if (mma34 && ok) {
      tc::tc_fence_after();
      const int r = tid;
      const float gC = kChan ? a.gC[chunk * kD + r] : __expf(ell_s[kC - 1]);
      // 16 columns at a time; the next 16 columns' tensor-memory loads are in flight
      // while the current ones are converted and stored
      uint32_t x[2][16], y[2][16];
      tmem_ld16(lane_addr, x[0]);
      tmem_ld16(lane_addr + 128, y[0]);
      tmem_wait_ld_regs(x[0], y[0]);
#pragma unroll
      for (int k = 0; k < kD / 16; ++k) {
        const int cur = k & 1;
        if (k + 1 < kD / 16) {
          tmem_ld16(lane_addr + 16 * (k + 1), x[cur ^ 1]);
          tmem_ld16(lane_addr + 128 + 16 * (k + 1), y[cur ^ 1]);
        }
        const int cc = 16 * k;
        const int half = cc >> 6;
        uint8_t* bst = sm + (half ? kX : kTT);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int c8 = ((cc & 63) >> 3) + q;
          uint32_t wa[4], wb[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = cc + 8 * q + 2 * e;
            const float a0 = (r == c ? gC : 0.0f) - __uint_as_float(x[cur][8 * q + 2 * e]);
            const float a1 = (r == c + 1 ? gC : 0.0f) - __uint_as_float(x[cur][8 * q + 2 * e + 1]);
            wa[e] = tc::pack_bf16x2(a0, a1);
            wb[e] = tc::pack_bf16x2(__uint_as_float(y[cur][8 * q + 2 * e]),
                                    __uint_as_float(y[cur][8 * q + 2 * e + 1]));
          }
          *(uint4*)(sm + kScr + half * 16384 + swz(r, c8)) = make_uint4(wa[0], wa[1], wa[2], wa[3]);
          *(uint4*)(bst + swz(r, c8)) = make_uint4(wb[0], wb[1], wb[2], wb[3]);
        }
        if (k + 1 < kD / 16) tmem_wait_ld_regs(x[cur ^ 1], y[cur ^ 1]);
      }
      tc::fence_async_smem();
      tc::tc_fence_before();
      tc::bar_sync(1, 128);
      if (tid == 0) {
        const int y = (int)((P.bh * a.ab_chunk_stride + P.i) * kD);
        tc::tma_store_2d(&tmA, sm + kScr, 0, y);
        tc::tma_store_2d(&tmA, sm + kScr + 16384, 64, y);
        tc::tma_store_2d(&tmB, sm + kTT, 0, y);
        tc::tma_store_2d(&tmB, sm + kX, 64, y);
        tc::bulk_commit();
      }
    }
    // every reader of this chunk's shared and tensor memory is done
    tc::tc_fence_before();
    ok = tc::bar_all(1, 128, ok);
  }

  if (tid == 0) {
    tc::bulk_wait_all();
    // never leave the CTA with a copy in flight
    if (load_pending) tc::mbar_wait(&bars[0], load_parity, nullptr, 200000000ull);
    if (kh_pending) tc::mbar_wait(&bars[4], it & 1, nullptr, 200000000ull);
    if (kc_pending) tc::mbar_wait(&bars[5], ph5 & 1, nullptr, 200000000ull);
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (warp == 0) tc::tmem_dealloc(tm, 256);
  if (tid == 0 && *abort_s) report_device_error(kErrMbarTimeout);
}

}  // namespace

// Transitions for bf16, d = 128 over [B,T,H,d] inputs (k, v) and [B,T,H] alpha/beta;
// with `chan` (channel-wise decay) over the prepared operands of every sub-chunk.
cudaError_t launch_transitions_tc(const TransArgs& t, cudaStream_t s, const ChanOperands* chan) {
  if (t.n_chunks <= 0) return cudaSuccess;
  const long HD = (long)t.H * kD;
  const long rows = (long)t.B * (t.in.sb / HD);  // B x tokens per sequence
  const long total = (long)t.B * t.H * t.n_chunks;
  const long ab_rows = (long)t.B * t.H * t.ab_chunk_stride * kD;
  // tile coordinates are 32-bit
  if (rows >= (1L << 31) || total * kC >= (1L << 31) || ab_rows >= (1L << 31)) return cudaErrorNotSupported;
  CUtensorMap tk, tv, twb, tub, ta, tb, tkh, tkc;
  cudaError_t e = cudaSuccess;
  if (chan != nullptr) {
    // Kt, Kh, Kc: [total chunks x 64 rows, 128] bf16
    e = make_tmap_2d(&tk, chan->Kt, kD, total * kC, kD * 2, 64, 64);
    if (e == cudaSuccess) e = make_tmap_2d(&tkh, chan->Kh, kD, total * kC, kD * 2, 64, 64);
    if (e == cudaSuccess) e = make_tmap_2d(&tkc, chan->Kc, kD, total * kC, kD * 2, 64, 64);
  } else {
    e = make_tmap_2d(&tk, t.in.k, HD, rows, HD * 2, 64, 64);
    tkh = tk;  // not used
    tkc = tk;
  }
  if (e == cudaSuccess) e = make_tmap_2d(&tv, t.in.v, HD, rows, HD * 2, 64, 64);
  // outputs that are not requested get a valid map that is never used
  const void* wb = t.Wb ? (const void*)t.Wb : t.in.k;
  const void* ub = t.Ub ? (const void*)t.Ub : t.in.k;
  const bool has_ab = t.A != nullptr && t.Bm != nullptr && t.ab_chunk_stride > 0;
  const void* ab = has_ab ? t.A : t.in.k;
  const void* bb = has_ab ? t.Bm : t.in.k;
  const long wu_rows = t.Wb ? total * kC : 64;
  const long ab_map_rows = has_ab ? ab_rows : 128;
  if (e == cudaSuccess) e = make_tmap_2d(&twb, wb, kD, wu_rows, kD * 2, 64, 64);
  if (e == cudaSuccess) e = make_tmap_2d(&tub, ub, kD, wu_rows, kD * 2, 64, 64);
  if (e == cudaSuccess) e = make_tmap_2d(&ta, ab, kD, ab_map_rows, kD * 2, 64, 128);
  if (e == cudaSuccess) e = make_tmap_2d(&tb, bb, kD, ab_map_rows, kD * 2, 64, 128);
  if (e != cudaSuccess) return e;
  TransTcArgs a;
  a.B = t.B;
  a.H = t.H;
  a.T = (int)(t.in.sb / HD);  // tokens per sequence in the input layout
  a.N = t.n_chunks;
  a.total = total;
  a.sb_a = t.in.ab;
  a.sh_a = t.in.ah;
  a.st_a = t.in.at;
  // beta is [B,T,H]; with a decay per channel the alpha strides carry a factor d
  const long bdiv = t.in.alpha_vec ? kD : 1;
  a.sb_b = t.in.ab / bdiv;
  a.sh_b = t.in.ah / bdiv;
  a.st_b = t.in.at / bdiv;
  a.alpha = t.in.alpha;
  a.beta = t.in.beta;
  a.has_ab = has_ab;
  a.ab_chunk_stride = t.ab_chunk_stride;
  a.has_wu = t.Wb != nullptr && t.Ub != nullptr;
  a.ell = chan != nullptr ? nullptr : t.ell;
  a.gC = chan != nullptr ? chan->gC : nullptr;
  const size_t smem = 1024 + kSmemUsed;
  const long grid = total < 2L * num_sms() ? total : 2L * num_sms();
  if (chan != nullptr) {
    e = cudaFuncSetAttribute(transitions_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    transitions_tc_kernel<true><<<(unsigned)grid, 128, smem, s>>>(tk, tv, twb, tub, ta, tb, tkh, tkc, a);
    return cudaGetLastError();
  }
  e = cudaFuncSetAttribute(transitions_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  transitions_tc_kernel<false><<<(unsigned)grid, 128, smem, s>>>(tk, tv, twb, tub, ta, tb, tkh, tkc, a);
  return cudaGetLastError();
}

}  // namespace hla
