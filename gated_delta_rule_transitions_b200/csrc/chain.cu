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
// Tensor-core version (bf16, d = 128): chain_pipe_kernel below, a persistent CTA per
// SM with a TMA-fed ring; the running product X is the bf16 A operand of
//   D = X A_k      (tcgen05.mma, M = N = K = 128, float32 accumulator in TMEM).
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

// Tensor-core chains, persistent and pipelined.  One CTA per SM walks the jobs
// blockIdx.x, blockIdx.x + gridDim.x, ... with three roles:
//   warp 0       TMA producer: per job the starting matrix X0, then per step the
//                right factor A_k and (B-chains, advance) B_k, into a 3-stage ring of
//                64 KiB items that runs ahead across job boundaries;
//   warp 1       TMEM allocation and the MMA issuer (one lane): step 0 multiplies X0
//                straight from shared memory (SS form), later steps take the running
//                product from tensor memory (TS form), D = X A_k into TMEM;
//   warps 2-5    epilogue, one row v per thread: D + B_k (B_k rows read from the
//                ring), rounded to bf16, written back as the next operand and, where
//                the chain emits, to global memory.
// Barriers: full/empty per stage (empty: the MMA's commit and the four epilogue
// warps), mma_done per step, op_ready per step (the operand is written and D has
// been read).  The epilogue releases a stage only after it has seen the step's
// mma_done, so every commit of an earlier use of that stage has arrived before.
// All waits are bounded.
constexpr int kPStages = 3;
constexpr int kPStage = 2 * kTile;  // X0 or A_k, then B_k: 64 KiB
constexpr int kPThreads = 192;

template <bool kAdvance>
__global__ void __launch_bounds__(kPThreads, 1)
    chain_pipe_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const __grid_constant__ CUtensorMap tmX, ChainArgs a, long njobs) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* ring = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* full = (uint64_t*)(ring + kPStages * kPStage);
  uint64_t* empty = full + kPStages;
  uint64_t* mma_done = empty + kPStages;
  uint64_t* op_ready = mma_done + 1;
  uint64_t* fin_bar = op_ready + 1;
  uint32_t* tmem_s = (uint32_t*)(fin_bar + 1);
  volatile int* abort_s = (volatile int*)(tmem_s + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int st = 0; st < kPStages; ++st) {
      tc::mbar_init(&full[st], 1);
      tc::mbar_init(&empty[st], 1 + 4);
    }
    tc::mbar_init(mma_done, 1);
    tc::mbar_init(op_ready, 4);
    tc::mbar_init(fin_bar, 1);
    *abort_s = 0;
    tc::mbar_fence_init();
    tc::fence_async_smem();
  }
  if (warp == 1) tc::tmem_alloc(tmem_s, 256);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tm = *tmem_s;  // columns 0-127: D (float32); 128-191: operand (bf16 pairs)

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      tc::tma_prefetch_desc(&tmA);
      tc::tma_prefetch_desc(&tmB);
      tc::tma_prefetch_desc(&tmX);
      long s = 0;
      bool ok = true;
      for (long blk = blockIdx.x; blk < njobs && ok; blk += gridDim.x) {
        ChainJob jb;
        if (!chain_job<kAdvance>(a, blk, kD, jb)) continue;
        const CUtensorMap* xmap = kAdvance ? &tmX : (jb.x_is_B ? &tmB : &tmA);
        for (int item = 0; item <= jb.nsteps; ++item, ++s) {
          const int st = (int)(s % kPStages);
          if (s >= kPStages && !tc::mbar_wait(&empty[st], (uint32_t)((s / kPStages) - 1) & 1, abort_s)) {
            ok = false;
            break;
          }
          uint8_t* dst = ring + st * kPStage;
          if (item == 0) {
            const int row = (int)(jb.x0 / kD);  // X0 starts at row (matrix index) x 128
            tc::mbar_arrive_expect_tx(&full[st], kTile);
            tc::tma_load_2d(dst, xmap, 0, row, &full[st]);
            tc::tma_load_2d(dst + kHalf, xmap, 64, row, &full[st]);
          } else {
            const int row = (int)((jb.sub0 + item - 1) * kD);
            tc::mbar_arrive_expect_tx(&full[st], jb.addB ? 2 * kTile : kTile);
            tc::tma_load_2d(dst, &tmA, 0, row, &full[st]);
            tc::tma_load_2d(dst + kHalf, &tmA, 64, row, &full[st]);
            if (jb.addB) {
              tc::tma_load_2d(dst + kTile, &tmB, 0, row, &full[st]);
              tc::tma_load_2d(dst + kTile + kHalf, &tmB, 64, row, &full[st]);
            }
          }
        }
      }
      if (*abort_s)  // never leave the CTA with copies in flight
        for (long t = s - kPStages > 0 ? s - kPStages : 0; t < s; ++t)
          tc::mbar_wait(&full[t % kPStages], (uint32_t)(t / kPStages) & 1, nullptr, 200000000ull);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      long s = 0, step = 0;
      bool ok = true;
      for (long blk = blockIdx.x; blk < njobs && ok; blk += gridDim.x) {
        ChainJob jb;
        if (!chain_job<kAdvance>(a, blk, kD, jb)) continue;
        const int xs = (int)(s % kPStages);
        if (!tc::mbar_wait(&full[xs], (uint32_t)(s / kPStages) & 1, abort_s)) break;
        ++s;
        for (int k = 0; k < jb.nsteps; ++k, ++s, ++step) {
          const int st = (int)(s % kPStages);
          if (!tc::mbar_wait(&full[st], (uint32_t)(s / kPStages) & 1, abort_s) ||
              (step > 0 && !tc::mbar_wait(op_ready, (uint32_t)(step - 1) & 1, abort_s))) {
            ok = false;
            break;
          }
          tc::tc_fence_after();
          const uint32_t b_base = tc::smem_u32(ring + st * kPStage);
          if (k == 0) {
            const uint32_t a_base = tc::smem_u32(ring + xs * kPStage);
#pragma unroll
            for (int ks = 0; ks < kD / 16; ++ks) {
              const uint64_t ad = tc::sdesc_sw128(a_base + (ks >> 2) * kHalf + (ks & 3) * 32, 16, 1024);
              const uint64_t bd = tc::sdesc_sw128(b_base + ks * 2048, kHalf, 1024);
              tc::mma_ss(tm, ad, bd, kIdesc, ks > 0 ? 1u : 0u);
            }
          } else {
#pragma unroll
            for (int ks = 0; ks < kD / 16; ++ks) {
              const uint64_t bd = tc::sdesc_sw128(b_base + ks * 2048, kHalf, 1024);
              tc::mma_ts(tm, tm + 128u + 8u * ks, bd, kIdesc, ks > 0 ? 1u : 0u);
            }
          }
          tc::mma_commit(mma_done);
          if (k == 0) tc::mma_commit(&empty[xs]);
          tc::mma_commit(&empty[st]);
        }
      }
      // every MMA issued by this thread completes before tensor memory is freed
      tc::mma_commit(fin_bar);
      tc::mbar_wait(fin_bar, 0, nullptr, 200000000ull);
    }
    __syncwarp();
  } else {
    // ---------------- epilogue: warps 2-5, one row per thread ----------------
    const int q = warp & 3;  // TMEM lane quarter of this warp
    const int v = 32 * q + lane;
    const uint32_t lane_off = (uint32_t)(32 * q) << 16;
    long s = 0, step = 0;
    bool ok = true;
    for (long blk = blockIdx.x; blk < njobs && ok; blk += gridDim.x) {
      ChainJob jb;
      if (!chain_job<kAdvance>(a, blk, kD, jb)) continue;
      __nv_bfloat16* odst = kAdvance ? (__nv_bfloat16*)a.S : (__nv_bfloat16*)(jb.x_is_B ? a.Bout : a.Aout);
      const int xs = (int)(s % kPStages);
      ++s;
      for (int k = 0; k < jb.nsteps; ++k, ++s, ++step) {
        const int st = (int)(s % kPStages);
        ok = tc::bar_all(1, 128, tc::mbar_wait(mma_done, (uint32_t)step & 1, abort_s) &&
                                     tc::mbar_wait(&full[st], (uint32_t)(s / kPStages) & 1, abort_s));
        if (!ok) break;
        tc::tc_fence_after();
        if (k == 0 && lane == 0) tc::mbar_arrive(&empty[xs]);  // X0 has been multiplied
        const bool last = k + 1 == jb.nsteps;
        const bool emit = kAdvance || last;
        uint4* orow = emit ? (uint4*)(odst + jb.out0 + (kAdvance ? (long)k * kD * kD : 0) + (long)v * kD) : nullptr;
        const uint8_t* bst = ring + st * kPStage + kTile;  // B_k of this step (two 64-column boxes)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t dr[32];
          tc::tmem_ld32(tm + lane_off + 32u * c, dr);
          tc::tmem_wait_ld();
          uint32_t w[16];
          if (jb.addB) {
            const uint8_t* brow = bst + (c >> 1) * kHalf + v * 128;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int c8 = (c & 1) * 4 + e;
              const uint4 bq = *(const uint4*)(brow + ((c8 ^ (v & 7)) << 4));
              const uint32_t bw[4] = {bq.x, bq.y, bq.z, bq.w};
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                const float2 bb = tc::bf16x2_to_float2(bw[u]);
                const int i = 4 * e + u;
                w[i] = tc::pack_bf16x2(__uint_as_float(dr[2 * i]) + bb.x, __uint_as_float(dr[2 * i + 1]) + bb.y);
              }
            }
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) w[i] = tc::pack_bf16x2(__uint_as_float(dr[2 * i]), __uint_as_float(dr[2 * i + 1]));
          }
          if (!last) tc::tmem_st16(tm + lane_off + 128u + 16u * c, w);
          if (emit) {
#pragma unroll
            for (int e = 0; e < 4; ++e) orow[4 * c + e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
          }
        }
        if (!last) tc::tmem_wait_st();
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          tc::mbar_arrive(op_ready);   // operand written, D read
          tc::mbar_arrive(&empty[st]);  // B_k read
        }
      }
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (warp == 1) tc::tmem_dealloc(tm, 256);
  if (threadIdx.x == 0 && *abort_s) report_device_error(kErrMbarTimeout);
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
cudaError_t launch_tc(const ChainArgs& a, long jobs, cudaStream_t s) {
  // TMA row coordinates are 32-bit
  const long rows = (long)a.B * a.H * a.sub_stride * kD;
  const long srows = (long)a.B * a.H * a.Nsub * kD;
  if (rows >= (1L << 31) || (kAdvance && srows >= (1L << 31))) return cudaErrorInvalidValue;
  CUtensorMap tmA, tmB, tmX;
  cudaError_t e = make_tmap_rows128(&tmA, a.Asub, rows);
  if (e == cudaSuccess) e = make_tmap_rows128(&tmB, a.Bsub, rows);
  if (e == cudaSuccess) e = kAdvance ? make_tmap_rows128(&tmX, a.S, srows) : make_tmap_rows128(&tmX, a.Asub, rows);
  if (e != cudaSuccess) return e;
  const size_t smem = 1024 + kPStages * kPStage + 128;
  e = cudaFuncSetAttribute(chain_pipe_kernel<kAdvance>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long grid = jobs < num_sms() ? jobs : num_sms();
  chain_pipe_kernel<kAdvance><<<(unsigned)grid, kPThreads, smem, s>>>(tmA, tmB, tmX, a, jobs);
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
