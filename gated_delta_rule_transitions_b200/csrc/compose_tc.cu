// Gated composition on the 5th-generation tensor cores (tcgen05 + TMEM + TMA),
// bf16 operands, float32 state.  d = 128, C = 64.
//
// HLA summary page, "Methodology in Plain English" paras. 3-4: for query chunk i,
//   S <- 0;  for j in active(i), ascending:  S <- S + g_ij ((S A_j + B_j) - S)
// and a chunk below the threshold is skipped (it is not in active(i)).
//
// One CTA runs three query chunks ("chains") of one head; every step of the merged
// active lists brings A_j and B_j once (TMA, 128-byte swizzle, 3-stage ring) for all
// three.  Each chain step is one MMA
//     D_k += Aop_k x A_j     (M = 128 rows v, N = 128 columns c, K = 128)
// with the float32 master state pre-scaled in tensor memory, D_k = (1-g) S, and the
// bf16 operand Aop_k = g S (tensor memory for chains 0 and 1, shared memory for
// chain 2 -- tensor memory holds three float32 states and two operands).  The
// epilogue of the chain then adds g B_j[v][c] (S_new) and prepares the chain's next
// active step: D_k <- (1 - g_next) S_new, Aop_k <- bf16(g_next S_new).  After a
// chain's last active step S_new is written to S_in (bf16, [v][c]).  With three
// chains the tensor core has two other chains' MMAs to run while one chain's
// epilogue and hand-offs are in flight.
//
// Warp roles: warp 0 TMA producer (walks the merged lists, publishes each step's
// schedule entry beside its stage), warp 1 TMEM allocator + MMA issuer, warps 2-5 /
// 6-9 / 10-13 epilogue of chain 0 / 1 / 2 (lane quarter = warp % 4, all 128 columns
// in 32-column chunks with the next chunk's TMEM load in flight).  All waits are
// bounded (about 2 s, then a device error word is set and the CTA exits cleanly).
#include "common.cuh"
#include "kernels.cuh"
#include "tc_common.cuh"

namespace hla {

HLA_DEFINE_ERROR_WORD(compose_tc)

namespace {

constexpr int kD = 128;
constexpr int kNC = 3;                           // chains per CTA
constexpr int kStages = 3;
constexpr int kStageBytes = 2 * kD * kD * 2;     // A_j + B_j, bf16
constexpr int kHalfBytes = kD * 64 * 2;          // one 64-column box
constexpr int kOpSmemBytes = kD * kD * 2;        // chain 2's bf16 operand (K-major, 128-byte swizzle)
constexpr int kEpiWarps = 4;                     // per chain
constexpr int kThreads = (2 + kNC * kEpiWarps) * 32;
constexpr uint32_t kIdescTS = tc::idesc_bf16_f32(128, 128, /*a_mn=*/0, /*b_mn=*/1);
constexpr uint32_t kIdescSS = tc::idesc_bf16_f32(128, 128, /*a_mn=*/0, /*b_mn=*/1);

struct ComposeTcArgs {
  int BH, N;
  long ab_chunk_stride;
  const int32_t* act_idx;
  const float* act_g;
  const int32_t* act_cnt;
  __nv_bfloat16* S_in;  // [B,H,N,d,d] bf16, row v, column c
};

// Walks the merged ascending active lists of the chains (producer only).
struct Sched {
  const int32_t* idx[kNC];
  const float* g[kNC];
  int cnt[kNC];
  int p[kNC];
  int j;
  bool act[kNC];

  __device__ void init(const ComposeTcArgs& a, int bh, const int (&i)[kNC]) {
    for (int k = 0; k < kNC; ++k) {
      p[k] = 0;
      if (i[k] >= 0) {
        const long row = (long)bh * a.N + i[k];
        idx[k] = a.act_idx + row * a.N;
        g[k] = a.act_g + row * a.N;
        cnt[k] = a.act_cnt[row];
      } else {
        idx[k] = nullptr;
        g[k] = nullptr;
        cnt[k] = 0;
      }
    }
  }
  __device__ bool next() {
    int jj[kNC];
    j = 0x7FFFFFFF;
    for (int k = 0; k < kNC; ++k) {
      jj[k] = p[k] < cnt[k] ? idx[k][p[k]] : 0x7FFFFFFF;
      j = min(j, jj[k]);
    }
    if (j == 0x7FFFFFFF) return false;
    for (int k = 0; k < kNC; ++k) act[k] = jj[k] == j;
    return true;
  }
  __device__ void advance() {
    for (int k = 0; k < kNC; ++k)
      if (act[k]) ++p[k];
  }
};

template <typename T>
__device__ __forceinline__ T pick(const T (&a)[kNC], int k) {
  return k == 0 ? a[0] : (k == 1 ? a[1] : a[2]);
}

// One step of the merged schedule, published by the producer next to its stage.
struct StepInfo {
  int j;          // chunk index; -1 ends the schedule
  int flags;      // bit k: chain k active; bit 4+k: first step; bit 8+k: last step
  int p[kNC];     // index of this step in each chain's active list
  float g[kNC];   // gates at this step
  float gn[kNC];  // gates at each chain's next active step (0 if none)
};

__global__ void __launch_bounds__(kThreads, 1)
    compose_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      ComposeTcArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* ring = smem;                                // kStages x [A h0 | A h1 | B h0 | B h1]
  uint8_t* op_smem = smem + kStages * kStageBytes;     // chain 2's operand, [kb][128 rows][128 B]
  uint64_t* bars = (uint64_t*)(op_smem + kOpSmemBytes);
  uint64_t* full = bars;                         // [kStages]
  uint64_t* empty = bars + kStages;              // [kStages]
  uint64_t* mma_done = bars + 2 * kStages;       // [kNC]
  uint64_t* op_ready = mma_done + kNC;           // [kNC]
  uint64_t* final_bar = op_ready + kNC;          // [1]
  StepInfo* info = (StepInfo*)(final_bar + 1);   // [kStages]
  uint32_t* tmem_base_s = (uint32_t*)(info + kStages);
  volatile int* abort_s = (volatile int*)(tmem_base_s + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int trip = blockIdx.x / a.BH;
  const int bh = blockIdx.x % a.BH;
  int chains[kNC];
  for (int k = 0; k < kNC; ++k) chains[k] = a.N - 1 - kNC * trip - k;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1 + kNC * kEpiWarps);  // MMA commit + lane 0 of every epilogue warp
    }
    for (int k = 0; k < kNC; ++k) {
      tc::mbar_init(&mma_done[k], 1);
      tc::mbar_init(&op_ready[k], kEpiWarps);
    }
    tc::mbar_init(final_bar, 1);
    *abort_s = 0;
    tc::mbar_fence_init();
    tc::fence_async_smem();
  }
  if (warp == 0 && lane == 0) {
    tc::tma_prefetch_desc(&tmA);
    tc::tma_prefetch_desc(&tmB);
  }
  if (warp == 1) tc::tmem_alloc(tmem_base_s, 512);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tbase = *tmem_base_s;
  // tensor memory: D_k at columns 128 k (k < 3), Aop_0 at 384, Aop_1 at 448

  if (warp == 0) {
    // ---------------- TMA producer (lane 0) ----------------
    if (lane == 0) {
      Sched sc;
      sc.init(a, bh, chains);
      int s = 0;
      bool ok = true;
      while (sc.next()) {
        const int st = s % kStages;
        if (s >= kStages && !tc::mbar_wait(&empty[st], ((s / kStages) - 1) & 1, abort_s)) {
          ok = false;
          break;
        }
        StepInfo e;
        e.j = sc.j;
        e.flags = 0;
        for (int k = 0; k < kNC; ++k) {
          const bool act = sc.act[k];
          const bool last = act && sc.p[k] + 1 == sc.cnt[k];
          e.flags |= (act ? 1 : 0) << k;
          e.flags |= ((act && sc.p[k] == 0) ? 1 : 0) << (4 + k);
          e.flags |= (last ? 1 : 0) << (8 + k);
          e.p[k] = sc.p[k];
          e.g[k] = act ? sc.g[k][sc.p[k]] : 0.0f;
          e.gn[k] = (act && !last) ? sc.g[k][sc.p[k] + 1] : 0.0f;
        }
        info[st] = e;
        tc::mbar_arrive_expect_tx(&full[st], kStageBytes);  // releases info[st]
        const int row = (int)(((long)bh * a.ab_chunk_stride + sc.j) * kD);
        uint8_t* dst = ring + st * kStageBytes;
        tc::tma_load_2d(dst, &tmA, 0, row, &full[st]);
        tc::tma_load_2d(dst + kHalfBytes, &tmA, 64, row, &full[st]);
        tc::tma_load_2d(dst + 2 * kHalfBytes, &tmB, 0, row, &full[st]);
        tc::tma_load_2d(dst + 3 * kHalfBytes, &tmB, 64, row, &full[st]);
        sc.advance();
        ++s;
      }
      if (ok) {
        // end marker: a stage phase with no data
        const int st = s % kStages;
        if (s < kStages || tc::mbar_wait(&empty[st], ((s / kStages) - 1) & 1, abort_s)) {
          info[st].j = -1;
          tc::mbar_arrive(&full[st]);
        }
      }
      if (*abort_s) {
        // never leave the CTA with copies in flight
        for (int t = max(0, s - kStages); t < s; ++t)
          tc::mbar_wait(&full[t % kStages], (t / kStages) & 1, nullptr, 200000000ull);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer (lane 0) ----------------
    if (lane == 0) {
      const uint32_t op_s = tc::smem_u32(op_smem);
      for (int s = 0;; ++s) {
        const int st = s % kStages;
        if (!tc::mbar_wait(&full[st], (s / kStages) & 1, abort_s)) break;
        const StepInfo e = info[st];
        if (e.j < 0) break;
        tc::tc_fence_after();
        const uint32_t b_base = tc::smem_u32(ring + st * kStageBytes);
        bool ok = true;
        for (int k = 0; k < kNC; ++k) {
          if (!((e.flags >> k) & 1) || ((e.flags >> (4 + k)) & 1)) continue;
          if (!tc::mbar_wait(&op_ready[k], (e.p[k] - 1) & 1, abort_s)) {
            ok = false;
            break;
          }
          tc::tc_fence_after();
          const uint32_t d_t = tbase + 128u * k;
          if (k < 2) {
            const uint32_t a_t = tbase + 384u + 64u * k;
#pragma unroll
            for (int ks = 0; ks < kD / 16; ++ks)
              tc::mma_ts(d_t, a_t + 8u * ks, tc::sdesc_sw128(b_base + ks * 2048, kHalfBytes, 1024), kIdescTS, 1u);
          } else {
#pragma unroll
            for (int ks = 0; ks < kD / 16; ++ks)
              tc::mma_ss(d_t, tc::sdesc_sw128(op_s + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024),
                         tc::sdesc_sw128(b_base + ks * 2048, kHalfBytes, 1024), kIdescSS, 1u);
          }
          tc::mma_commit(&mma_done[k]);
        }
        if (!ok) break;
        tc::mma_commit(&empty[st]);
      }
      // all MMAs issued by this thread complete before the CTA frees tensor memory
      tc::mma_commit(final_bar);
      tc::mbar_wait(final_bar, 0, nullptr, 200000000ull);
    }
    __syncwarp();
  } else {
    // ------- epilogue: chain k (4 warps, 128 threads, named barrier 1 + k) -------
    const int k = (warp - 2) / kEpiWarps;
    const int bar_id = 1 + k;
    const int q = warp & 3;
    const int v = 32 * q + lane;
    const uint32_t lane_off = (uint32_t)(32 * q) << 16;
    const uint32_t d_addr = tbase + lane_off + 128u * k;
    const uint32_t a_addr = tbase + lane_off + 384u + 64u * (k & 1);
    const int chain = chains[0] * (k == 0) + chains[1] * (k == 1) + chains[2] * (k == 2);
    const int cnt = chain >= 0 ? a.act_cnt[(long)bh * a.N + chain] : 0;
    __nv_bfloat16* out_row = chain >= 0 ? a.S_in + ((long)bh * a.N + chain) * kD * kD + (long)v * kD : nullptr;
    if (chain >= 0 && cnt == 0)  // a chain with nothing active has S_in = 0
      for (int e = 0; e < 16; ++e) ((uint4*)out_row)[e] = make_uint4(0u, 0u, 0u, 0u);
    for (int s = 0;; ++s) {
      const int st = s % kStages;
      const bool w = tc::mbar_wait(&full[st], (s / kStages) & 1, abort_s);
      const int jv = w ? ((volatile StepInfo*)info)[st].j : 0;
      // one vote per step: stop at the end marker or on a timeout anywhere
      if (tc::bar_any(bar_id, 32 * kEpiWarps, !w || *abort_s != 0 || jv < 0)) break;
      const StepInfo e = info[st];
      const bool act = (e.flags >> k) & 1;
      const bool last = (e.flags >> (8 + k)) & 1;
      if (act) {
        const bool first = (e.flags >> (4 + k)) & 1;
        const float g = pick(e.g, k);
        const float gn = pick(e.gn, k);
        const int pk = pick(e.p, k);
        const float keep = 1.0f - gn;
        if (!first) {
          tc::mbar_wait(&mma_done[k], (pk - 1) & 1, abort_s);
          tc::tc_fence_after();
        }
        const uint8_t* brow = ring + st * kStageBytes + 2 * kHalfBytes + v * 128;
        const float2 g2 = make_float2(g, g);
        const float2 gn2 = make_float2(gn, gn), keep2 = make_float2(keep, keep);
        uint32_t da[32], db[32];
        if (!first) {
          tc::tmem_ld32(d_addr, da);
          tc::tmem_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) da[i] = 0u;
        }
        // 32 columns: x = d + g b; either S_in, or (1-g') x back to D and g' x to the operand
        auto chunk = [&](uint32_t(&d)[32], int cc) {
          const uint8_t* bp = brow + (cc >> 6) * kHalfBytes;
          uint32_t bw[16];
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            const int c8 = ((cc & 63) >> 3) + c4;
            const uint4 w4 = *(const uint4*)(bp + ((c8 ^ (v & 7)) << 4));
            bw[4 * c4 + 0] = w4.x;
            bw[4 * c4 + 1] = w4.y;
            bw[4 * c4 + 2] = w4.z;
            bw[4 * c4 + 3] = w4.w;
          }
          uint32_t op[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float2 xv = tc::fma2(g2, tc::bf16x2_to_float2(bw[i]),
                                       make_float2(__uint_as_float(d[2 * i]), __uint_as_float(d[2 * i + 1])));
            if (last) {
              op[i] = tc::pack_bf16x2(xv.x, xv.y);
            } else {
              const float2 o = tc::mul2(gn2, xv);
              const float2 nn = tc::mul2(keep2, xv);
              op[i] = tc::pack_bf16x2(o.x, o.y);
              d[2 * i] = __float_as_uint(nn.x);
              d[2 * i + 1] = __float_as_uint(nn.y);
            }
          }
          if (last) {
            uint4* out = (uint4*)(out_row + cc);
#pragma unroll
            for (int i = 0; i < 4; ++i) out[i] = make_uint4(op[4 * i], op[4 * i + 1], op[4 * i + 2], op[4 * i + 3]);
          } else {
            tc::tmem_st32(d_addr + cc, d);
            if (k < 2) {
              tc::tmem_st16(a_addr + cc / 2, op);
            } else {
              // K-major operand row v: K block cc/64, 16-byte chunks swizzled by v
              uint8_t* orow = op_smem + (cc >> 6) * 16384 + v * 128;
#pragma unroll
              for (int c4 = 0; c4 < 4; ++c4) {
                const int c8 = ((cc & 63) >> 3) + c4;
                *(uint4*)(orow + ((c8 ^ (v & 7)) << 4)) =
                    make_uint4(op[4 * c4], op[4 * c4 + 1], op[4 * c4 + 2], op[4 * c4 + 3]);
              }
            }
          }
        };
        // four 32-column chunks; the next chunk's load is in flight during each
        if (!first) tc::tmem_ld32(d_addr + 32, db);
        chunk(da, 0);
        if (!first) {
          tc::tmem_wait_ld();
          tc::tmem_ld32(d_addr + 64, da);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) db[i] = 0u;
        }
        chunk(db, 32);
        if (!first) {
          tc::tmem_wait_ld();
          tc::tmem_ld32(d_addr + 96, db);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) da[i] = 0u;
        }
        chunk(da, 64);
        if (!first) {
          tc::tmem_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) db[i] = 0u;
        }
        chunk(db, 96);
        tc::tmem_wait_st();
        if (k == 2) tc::fence_async_smem();
        tc::tc_fence_before();
      }
      __syncwarp();
      if (lane == 0) {
        if (act && !last) tc::mbar_arrive(&op_ready[k]);
        tc::mbar_arrive(&empty[st]);
      }
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (warp == 1) tc::tmem_dealloc(tbase, 512);
  if (threadIdx.x == 0 && *abort_s) report_device_error(kErrMbarTimeout);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)p;
  }
  return fn;
}

}  // namespace

// 2-D bf16 tensor map, `inner` elements per row, `rows` rows, 128-byte swizzle.
cudaError_t make_tmap_2d(CUtensorMap* m, const void* base, long inner, long rows, long row_stride_bytes,
                         int box_inner, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return cudaErrorNotSupported;
  cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)row_stride_bytes};
  cuuint32_t box[2] = {(cuuint32_t)box_inner, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// 2-D bf16 tensor map over `rows` rows of 128 elements, box 64 x 128, 128-byte swizzle.
cudaError_t make_tmap_rows128(CUtensorMap* m, const void* base, long rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return cudaErrorNotSupported;
  cuuint64_t dims[2] = {128, (cuuint64_t)rows};
  cuuint64_t strides[1] = {128 * 2};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t launch_compose_tc(const ComposeArgs& c, cudaStream_t s) {
  if (c.N <= 0) return cudaSuccess;
  if (c.ab_chunk_stride <= 0)  // no complete chunk: every composed state is zero
    return cudaMemsetAsync(c.S_in, 0, (size_t)c.B * c.H * c.N * kD * kD * sizeof(__nv_bfloat16), s);
  const long rows = (long)c.B * c.H * c.ab_chunk_stride * kD;
  CUtensorMap tmA, tmB;
  cudaError_t e = make_tmap_rows128(&tmA, c.A, rows);
  if (e != cudaSuccess) return e;
  e = make_tmap_rows128(&tmB, c.Bm, rows);
  if (e != cudaSuccess) return e;
  ComposeTcArgs a;
  a.BH = c.B * c.H;
  a.N = c.N;
  a.ab_chunk_stride = c.ab_chunk_stride;
  a.act_idx = c.act_idx;
  a.act_g = c.act_g;
  a.act_cnt = c.act_cnt;
  a.S_in = (__nv_bfloat16*)c.S_in;
  const size_t smem = 1024 + kStages * kStageBytes + kOpSmemBytes + 512;
  e = cudaFuncSetAttribute(compose_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int trips = (c.N + kNC - 1) / kNC;
  compose_tc_kernel<<<trips * a.BH, kThreads, smem, s>>>(tmA, tmB, a);
  return cudaGetLastError();
}

}  // namespace hla
