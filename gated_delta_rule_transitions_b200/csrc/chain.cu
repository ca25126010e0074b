// Affine chains between 64-token sub-chunks and chunks of C = 64 s tokens.
//
// HLA summary page, "Methodology in Plain English" para. 1: affine maps compose, so
// consecutive sub-chunks S -> S A_k + B_k compose into the chunk's own transition,
// and the state entering any sub-chunk follows from the state entering its chunk:
//   merge    A_i = A_{is} ... A_{is+s-1},
//            B_i = (...(B_{is} A_{is+1} + B_{is+1}) ...) A_{is+s-1} + B_{is+s-1};
//   advance  S_(i,k) = S_(i,k-1) A_{is+k-1} + B_{is+k-1} from S_(i,0) = S_in(i).
// The pages' default chunk is 256 tokens ("Main Findings", chunk-size ablation).  At
// C = 64 s the gates, the composition and the decode cache work on chunks, while the
// WY solve and the intra-chunk read-out keep their 64-token tiles.  Merging costs
// 2 (s - 1) d^3 multiply-adds per chunk, less than a WY solve over C tokens would.
//
// Tensor-core version (bf16, d = 128): one CTA of 4 warps per chain.  All s - 1
// right-hand factors A_k arrive by TMA at once (128-byte swizzle, as compose_tc reads
// them).  The running product X lives in tensor memory as the bf16 A operand of
//   D = X A_k      (tcgen05.mma, M = N = K = 128, float32 accumulator in TMEM)
// and each thread (one row) adds its row of B_k, rounds to bf16 and writes the next
// operand back to tensor memory and, where the chain emits, to global memory.
// CUDA-core version (float32 arithmetic, any storage type, d = 64 or 128): one CTA
// of 256 threads per chain, X in shared memory.
#include "common.cuh"
#include "kernels.cuh"
#include "tc_common.cuh"

namespace hla {

HLA_DEFINE_ERROR_WORD(chain_tc)

cudaError_t make_tmap_rows128(CUtensorMap* m, const void* base, long rows);

namespace {

constexpr int kD = 128;
constexpr int kTile = kD * kD * 2;  // 32 KiB: one 128 x 128 bf16 matrix
constexpr int kHalf = kD * 64 * 2;  // 16 KiB: one 64-column box
constexpr int kMaxSteps = 3;        // s <= 4
constexpr uint32_t kIdesc = tc::idesc_bf16_f32(128, 128, /*a_mn=*/0, /*b_mn=*/1);

// One chain: X0, then steps k = 0 .. nsteps-1 with right factor A_{sub0 + k} and
// (if add) B_{sub0 + k}; emits every step (advance) or only the last (merge).
struct ChainJob {
  long x0;      // element offset of X0 in its array
  long sub0;    // sub-chunk slot of step 0's factors (matrix index into Asub/Bsub)
  long out0;    // element offset of the first emitted matrix in the output array
  int nsteps;
  bool addB;
  bool x_is_B;  // merge: X0 is B_{is} (else A_{is}); output Bout (else Aout)
};

template <bool kAdvance>
__device__ __forceinline__ bool chain_job(const ChainArgs& a, long blk, int d, ChainJob& j) {
  const long dd = (long)d * d;
  if (kAdvance) {
    const int i = (int)(blk % a.N);
    const long bh = blk / a.N;
    const int base = i * a.s;
    j.nsteps = min(a.s, a.Nsub - base) - 1;
    if (j.nsteps <= 0) return false;
    j.x0 = (bh * a.Nsub + base) * dd;
    j.sub0 = bh * a.sub_stride + base;
    j.out0 = (bh * a.Nsub + base + 1) * dd;
    j.addB = true;
    j.x_is_B = false;
  } else {
    j.x_is_B = (blk & 1) != 0;
    const long job = blk >> 1;
    const int i = (int)(job % a.Nc);
    const long bh = job / a.Nc;
    const long first = bh * a.sub_stride + (long)i * a.s;
    j.nsteps = a.s - 1;
    j.x0 = first * dd;
    j.sub0 = first + 1;
    j.out0 = (bh * a.out_stride + i) * dd;
    j.addB = j.x_is_B;
  }
  return true;
}

template <bool kAdvance>
__global__ void __launch_bounds__(128) chain_tc_kernel(const __grid_constant__ CUtensorMap tmA, ChainArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* tma_bar = (uint64_t*)(sm + kMaxSteps * kTile);  // [kMaxSteps]
  uint64_t* mma_bar = tma_bar + kMaxSteps;
  uint64_t* fin_bar = mma_bar + 1;
  uint32_t* tmem_s = (uint32_t*)(fin_bar + 1);
  volatile int* abort_s = (volatile int*)(tmem_s + 1);

  ChainJob jb;
  if (!chain_job<kAdvance>(a, blockIdx.x, kD, jb)) return;  // uniform over the CTA
  const __nv_bfloat16* xsrc = kAdvance ? (const __nv_bfloat16*)a.S
                                       : (const __nv_bfloat16*)(jb.x_is_B ? a.Bsub : a.Asub);
  __nv_bfloat16* odst = kAdvance ? (__nv_bfloat16*)a.S : (__nv_bfloat16*)(jb.x_is_B ? a.Bout : a.Aout);
  const __nv_bfloat16* bsub = (const __nv_bfloat16*)a.Bsub;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  if (tid == 0) {
    for (int k = 0; k < kMaxSteps; ++k) tc::mbar_init(&tma_bar[k], 1);
    tc::mbar_init(mma_bar, 1);
    tc::mbar_init(fin_bar, 1);
    *abort_s = 0;
    tc::mbar_fence_init();
    tc::fence_async_smem();
  }
  if (warp == 0) tc::tmem_alloc(tmem_s, 256);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tm = *tmem_s;  // columns 0-127: D (float32); 128-191: X (bf16 pairs)

  if (tid == 0) {
    tc::tma_prefetch_desc(&tmA);
    for (int k = 0; k < jb.nsteps; ++k) {
      tc::mbar_arrive_expect_tx(&tma_bar[k], kTile);
      const int row = (int)((jb.sub0 + k) * kD);
      tc::tma_load_2d(sm + k * kTile, &tmA, 0, row, &tma_bar[k]);
      tc::tma_load_2d(sm + k * kTile + kHalf, &tmA, 64, row, &tma_bar[k]);
    }
  }
  // X0 row v -> the operand columns (32 bf16 columns = 16 TMEM columns per store)
  const int v = tid;
  const uint32_t lane_off = (uint32_t)(32 * warp) << 16;
  // (the tcgen05 instructions order memory accesses around them, so every global
  // load of a row is issued before the first of them)
  {
    const uint4* src = (const uint4*)(xsrc + jb.x0 + (long)v * kD);
    uint4 xq[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) xq[e] = src[e];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t w[16];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        w[4 * e + 0] = xq[4 * c + e].x;
        w[4 * e + 1] = xq[4 * c + e].y;
        w[4 * e + 2] = xq[4 * c + e].z;
        w[4 * e + 3] = xq[4 * c + e].w;
      }
      tc::tmem_st16(tm + lane_off + 128u + 16u * c, w);
    }
    tc::tmem_wait_st();
  }
  // row v of B for the next step, loaded while the product runs
  uint4 bq[16];
  const __nv_bfloat16* brow0 = bsub + jb.sub0 * kD * kD + (long)v * kD;
  if (jb.addB) {
#pragma unroll
    for (int e = 0; e < 16; ++e) bq[e] = ((const uint4*)brow0)[e];
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();

  bool ok = true;
  for (int k = 0; k < jb.nsteps; ++k) {
    if (tid == 0 && tc::mbar_wait(&tma_bar[k], 0, abort_s)) {
      tc::tc_fence_after();
      const uint32_t b_base = tc::smem_u32(sm + k * kTile);
#pragma unroll
      for (int ks = 0; ks < kD / 16; ++ks) {
        const uint64_t bd = tc::sdesc_sw128(b_base + ks * 2048, kHalf, 1024);
        tc::mma_ts(tm, tm + 128u + 8u * ks, bd, kIdesc, ks > 0 ? 1u : 0u);
      }
      tc::mma_commit(mma_bar);
    }
    ok = tc::bar_all(1, 128, tc::mbar_wait(mma_bar, k & 1, abort_s));
    if (!ok) break;
    tc::tc_fence_after();
    const bool last = k + 1 == jb.nsteps;
    const bool emit = kAdvance || last;
    uint4* orow = emit ? (uint4*)(odst + jb.out0 + (kAdvance ? (long)k * kD * kD : 0) + (long)v * kD) : nullptr;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t dr[32];
      tc::tmem_ld32(tm + lane_off + 32u * c, dr);
      tc::tmem_wait_ld();
      uint32_t w[16];
      if (jb.addB) {
        uint32_t bw[16];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          bw[4 * e + 0] = bq[4 * c + e].x;
          bw[4 * e + 1] = bq[4 * c + e].y;
          bw[4 * e + 2] = bq[4 * c + e].z;
          bw[4 * e + 3] = bq[4 * c + e].w;
        }
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float2 bb = tc::bf16x2_to_float2(bw[e]);
          w[e] = tc::pack_bf16x2(__uint_as_float(dr[2 * e]) + bb.x, __uint_as_float(dr[2 * e + 1]) + bb.y);
        }
      } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) w[e] = tc::pack_bf16x2(__uint_as_float(dr[2 * e]), __uint_as_float(dr[2 * e + 1]));
      }
      if (!last) tc::tmem_st16(tm + lane_off + 128u + 16u * c, w);
      if (emit) {
#pragma unroll
        for (int e = 0; e < 4; ++e) orow[4 * c + e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
      }
    }
    if (!last) {
      tc::tmem_wait_st();
      if (jb.addB) {  // the next step's row of B, in flight across the next product
        const uint4* bn = (const uint4*)(brow0 + (long)(k + 1) * kD * kD);
#pragma unroll
        for (int e = 0; e < 16; ++e) bq[e] = bn[e];
      }
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
  }
  if (tid == 0) {
    if (!ok)  // never leave the CTA with copies in flight
      for (int k = 0; k < jb.nsteps; ++k) tc::mbar_wait(&tma_bar[k], 0, nullptr, 200000000ull);
    // every MMA issued by this thread completes before tensor memory is freed
    tc::mma_commit(fin_bar);
    tc::mbar_wait(fin_bar, 0, nullptr, 200000000ull);
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (warp == 0) tc::tmem_dealloc(tm, 256);
  if (tid == 0 && *abort_s) report_device_error(kErrMbarTimeout);
}

// CUDA-core chain: X (float32) in shared memory; each thread owns an R x R block of
// the product, as in the CUDA-core composition.  Tab: storage of A/B; Tx: storage of
// X0 and of the emitted matrices.
template <int D, typename Tab, typename Tx, bool kAdvance>
__global__ void __launch_bounds__(256) chain_simt_kernel(ChainArgs a) {
  constexpr int R = D / 16;
  constexpr int DP = D + 1;
  extern __shared__ float X[];  // [D][DP]
  ChainJob jb;
  if (!chain_job<kAdvance>(a, blockIdx.x, D, jb)) return;
  const Tx* xsrc = kAdvance ? (const Tx*)a.S : (const Tx*)(jb.x_is_B ? a.Bsub : a.Asub);
  Tx* odst = kAdvance ? (Tx*)a.S : (Tx*)(jb.x_is_B ? a.Bout : a.Aout);
  const int tid = threadIdx.x;
  const int ty = tid >> 4, tx = tid & 15;
  for (int idx = tid; idx < D * D; idx += blockDim.x) {
    const int r = idx / D, c = idx - r * D;
    X[r * DP + c] = ldf(xsrc + jb.x0 + idx);
  }
  __syncthreads();
  for (int k = 0; k < jb.nsteps; ++k) {
    const Tab* A = (const Tab*)a.Asub + (jb.sub0 + k) * (long)D * D;
    const Tab* Bm = jb.addB ? (const Tab*)a.Bsub + (jb.sub0 + k) * (long)D * D : nullptr;
    float acc[R][R];
#pragma unroll
    for (int u = 0; u < R; ++u)
#pragma unroll
      for (int w = 0; w < R; ++w) acc[u][w] = 0.0f;
    for (int m = 0; m < D; ++m) {
      float xv[R], av[R];
#pragma unroll
      for (int u = 0; u < R; ++u) xv[u] = X[(ty * R + u) * DP + m];
#pragma unroll
      for (int w = 0; w < R; ++w) av[w] = ldf(A + (long)m * D + tx * R + w);
#pragma unroll
      for (int u = 0; u < R; ++u)
#pragma unroll
        for (int w = 0; w < R; ++w) acc[u][w] = fmaf(xv[u], av[w], acc[u][w]);
    }
    __syncthreads();
    const bool emit = kAdvance || k + 1 == jb.nsteps;
    Tx* out = odst + jb.out0 + (kAdvance ? (long)k * D * D : 0);
#pragma unroll
    for (int u = 0; u < R; ++u) {
      const int r = ty * R + u;
#pragma unroll
      for (int w = 0; w < R; ++w) {
        const int c = tx * R + w;
        const float x = acc[u][w] + (Bm != nullptr ? ldf(Bm + (long)r * D + c) : 0.0f);
        X[r * DP + c] = x;
        if (emit) stf(out + (long)r * D + c, x);
      }
    }
    __syncthreads();
  }
}

template <int D, typename Tab, typename Tx, bool kAdvance>
cudaError_t launch_simt(const ChainArgs& a, long blocks, cudaStream_t s) {
  const size_t smem = (size_t)D * (D + 1) * sizeof(float);
  auto k = chain_simt_kernel<D, Tab, Tx, kAdvance>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k<<<(unsigned)blocks, 256, smem, s>>>(a);
  return cudaGetLastError();
}

template <bool kAdvance>
cudaError_t launch_tc(const ChainArgs& a, long blocks, cudaStream_t s) {
  // TMA row coordinates are 32-bit
  const long rows = (long)a.B * a.H * a.sub_stride * kD;
  if (rows >= (1L << 31)) return cudaErrorInvalidValue;
  CUtensorMap tmA;
  cudaError_t e = make_tmap_rows128(&tmA, a.Asub, rows);
  if (e != cudaSuccess) return e;
  const size_t smem = 1024 + kMaxSteps * kTile + 64;
  e = cudaFuncSetAttribute(chain_tc_kernel<kAdvance>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  chain_tc_kernel<kAdvance><<<(unsigned)blocks, 128, smem, s>>>(tmA, a);
  return cudaGetLastError();
}

bool tc_shape(const ChainArgs& a) { return a.dtype == HLA_BF16 && a.d == kD; }

}  // namespace

cudaError_t launch_chain_merge(const ChainArgs& a, cudaStream_t s) {
  if (a.s < 2 || a.s - 1 > kMaxSteps) return cudaErrorInvalidValue;
  const long blocks = 2L * a.B * a.H * a.Nc;
  if (blocks <= 0) return cudaSuccess;
  if (tc_shape(a)) return launch_tc<false>(a, blocks, s);
  if (a.d == 128)
    return a.dtype == HLA_BF16 ? launch_simt<128, __nv_bfloat16, __nv_bfloat16, false>(a, blocks, s)
                               : launch_simt<128, float, float, false>(a, blocks, s);
  return a.dtype == HLA_BF16 ? launch_simt<64, __nv_bfloat16, __nv_bfloat16, false>(a, blocks, s)
                             : launch_simt<64, float, float, false>(a, blocks, s);
}

cudaError_t launch_chain_advance(const ChainArgs& a, cudaStream_t s) {
  if (a.s < 2 || a.s - 1 > kMaxSteps) return cudaErrorInvalidValue;
  const long blocks = (long)a.B * a.H * a.N;
  if (blocks <= 0 || a.Nsub <= 1) return cudaSuccess;
  if (tc_shape(a)) return launch_tc<true>(a, blocks, s);
  // CUDA-core path: S_in is float32
  if (a.d == 128)
    return a.dtype == HLA_BF16 ? launch_simt<128, __nv_bfloat16, float, true>(a, blocks, s)
                               : launch_simt<128, float, float, true>(a, blocks, s);
  return a.dtype == HLA_BF16 ? launch_simt<64, __nv_bfloat16, float, true>(a, blocks, s)
                             : launch_simt<64, float, float, true>(a, blocks, s);
}

}  // namespace hla
