// Gated composition on the 5th-generation tensor cores (tcgen05 + TMEM + TMA),
// bf16 operands, float32 state.  d = 128, C = 64.
//
// HLA summary page, "Methodology in Plain English" paras. 3-4: for query chunk i,
//   S <- 0;  for j in active(i), ascending:  S <- S + g_ij ((S A_j + B_j) - S)
// and a chunk below the threshold is skipped (it is not in active(i)).
//
// Representation.  The state of a query chunk ("chain") is kept in tensor memory as
// D = S / rho with a per-chain scalar rho, and B_j enters through its rank-C factors
// B_j = Ub_j^T (D K)_j.  For a step with gate g < 1, choosing rho' = (1 - g) rho gives
//   D' = D + [c1 D | c2 Ub_j^T] x [A_j ; (D K)_j],  c1 = g / (1-g),  c2 = c1 / rho,
// one accumulating MMA with K = d + C = 192 (A operand from tensor memory, B operand
// [A_j; (DK)_j] from shared memory); for g = 1 the same MMA without accumulation and
// c1 = 1, rho' = rho.  The epilogue therefore only reads D and writes the bf16 operand
// for the chain's next step (no read-modify-write of the float32 state and no
// elementwise B_j); rho is renormalised into D when it falls below 2^-30.  The first
// step of a chain (S = 0) is the MMA over the Ub^T part alone: D = B_j1, rho = g_1.
// After a chain's last step S_in = rho D is written (bf16, [v][c]).
//
// One CTA runs two chains of one head.  Warp 0: TMA producer walking the merged
// active lists (4-stage ring of A_j and (DK)_j, 128-byte swizzle; each stage carries
// the step's schedule entry).  Warp 1: TMEM allocator and MMA issuer.  Warps 2-9 and
// 10-17: epilogue of chain 0 and chain 1 (lane quarter = warp % 4, column half =
// ((warp - 2) % 8) / 4), so each chain's epilogue overlaps the other chain's MMA.
// All waits are bounded (about 2 s, then a device error word is set and the CTA
// exits cleanly).
#include "common.cuh"
#include "kernels.cuh"
#include "tc_common.cuh"

namespace hla {

HLA_DEFINE_ERROR_WORD(compose_tc)

namespace {

constexpr int kD = 128;
constexpr int kC = 64;
constexpr int kStages = 4;
constexpr int kABytes = kD * kD * 2;             // A_j, bf16 (two 64-column boxes)
constexpr int kHalfBytes = kD * 64 * 2;          // one 64-column box of A_j
constexpr int kDKBytes = kC * kD * 2;            // (DK)_j, bf16 (two 64-column boxes)
constexpr int kStageBytes = kABytes + kDKBytes;  // 48 KiB
constexpr int kThreads = 576;                    // producer, MMA, 2 x 8 epilogue warps
constexpr uint32_t kIdesc = tc::idesc_bf16_f32(128, 128, /*a_mn=*/0, /*b_mn=*/1);
constexpr uint32_t kOpCols = 96;                 // per-chain operand columns: 64 (c1 D) + 32 (c2 Ub^T)

struct ComposeTcArgs {
  int BH, N;
  long ab_chunk_stride;        // chunk stride of A_j
  const int32_t* act_idx;
  const float* act_g;
  const int32_t* act_cnt;
  const __nv_bfloat16* UT;     // [BH, N, d, C] Ub^T of each chunk
  __nv_bfloat16* S_in;         // [BH, N, d, d] bf16, row v, column c
};

// Walks the merged ascending active lists of the two chains (producer only).
struct Sched {
  const int32_t* idx[2];
  const float* g[2];
  int cnt[2];
  int p[2];
  int j;
  bool act[2];
  bool first[2];
  float gate[2];
  float gnext[2];
  int jnext[2];
  bool last[2];

  __device__ void init(const ComposeTcArgs& a, int bh, const int i[2]) {
    for (int k = 0; k < 2; ++k) {
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
    int j0 = p[0] < cnt[0] ? idx[0][p[0]] : 0x7FFFFFFF;
    int j1 = p[1] < cnt[1] ? idx[1][p[1]] : 0x7FFFFFFF;
    j = min(j0, j1);
    if (j == 0x7FFFFFFF) return false;
    const int jj[2] = {j0, j1};
    for (int k = 0; k < 2; ++k) {
      act[k] = jj[k] == j;
      first[k] = act[k] && p[k] == 0;
      gate[k] = act[k] ? g[k][p[k]] : 0.0f;
      last[k] = act[k] && p[k] + 1 == cnt[k];
      gnext[k] = (act[k] && !last[k]) ? g[k][p[k] + 1] : 0.0f;
      jnext[k] = (act[k] && !last[k]) ? idx[k][p[k] + 1] : 0;
    }
    return true;
  }
  __device__ void advance() {
    for (int k = 0; k < 2; ++k)
      if (act[k]) ++p[k];
  }
};

// One step of the merged schedule, published by the producer next to its stage.
struct StepInfo {
  int j;       // chunk index; -1 ends the schedule
  int flags;   // bit k: chain k active; bit 2+k: first step of chain k; bit 4+k: last step
  int p[2];    // index of this step in each chain's active list
  float g[2];  // gates at this step
  float gn[2]; // gates at each chain's next active step
  int jn[2];   // chunk of each chain's next active step
};

__global__ void __launch_bounds__(kThreads, 1)
    compose_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmDK,
                      ComposeTcArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* ring = smem;  // kStages x [A half0 | A half1 | DK half0 | DK half1]
  uint64_t* bars = (uint64_t*)(smem + kStages * kStageBytes);
  uint64_t* full = bars;                    // [kStages]
  uint64_t* empty = bars + kStages;         // [kStages]
  uint64_t* mma_done = bars + 2 * kStages;  // [2]
  uint64_t* op_ready = mma_done + 2;        // [2]
  uint64_t* final_bar = op_ready + 2;       // [1]
  StepInfo* info = (StepInfo*)(final_bar + 1);  // [kStages]
  uint32_t* tmem_base_s = (uint32_t*)(info + kStages);
  volatile int* abort_s = (volatile int*)(tmem_base_s + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int pair = blockIdx.x / a.BH;
  const int bh = blockIdx.x % a.BH;
  const int chains[2] = {a.N - 1 - 2 * pair, a.N - 2 - 2 * pair};

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1 + 16);  // MMA commit + lane 0 of every epilogue warp
    }
    for (int k = 0; k < 2; ++k) {
      tc::mbar_init(&mma_done[k], 1);
      tc::mbar_init(&op_ready[k], 8);   // lane 0 of every warp of the chain's group
    }
    tc::mbar_init(final_bar, 1);
    *abort_s = 0;
    tc::mbar_fence_init();
    tc::fence_async_smem();
  }
  if (warp == 0 && lane == 0) {
    tc::tma_prefetch_desc(&tmA);
    tc::tma_prefetch_desc(&tmDK);
  }
  if (warp == 1) tc::tmem_alloc(tmem_base_s, 512);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tbase = *tmem_base_s;

  if (warp == 0) {
    // ---------------- TMA producer (lane 0): walks the merged lists ----------------
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
        for (int k = 0; k < 2; ++k) {
          e.flags |= (sc.act[k] ? 1 : 0) << k;
          e.flags |= (sc.first[k] ? 1 : 0) << (2 + k);
          e.flags |= (sc.last[k] ? 1 : 0) << (4 + k);
          e.p[k] = sc.p[k];
          e.g[k] = sc.gate[k];
          e.gn[k] = sc.gnext[k];
          e.jn[k] = sc.jnext[k];
        }
        info[st] = e;
        tc::mbar_arrive_expect_tx(&full[st], kStageBytes);  // releases info[st]
        const int rowA = (int)(((long)bh * a.ab_chunk_stride + sc.j) * kD);
        const int rowK = (int)(((long)bh * a.N + sc.j) * kC);
        uint8_t* dst = ring + st * kStageBytes;
        tc::tma_load_2d(dst, &tmA, 0, rowA, &full[st]);
        tc::tma_load_2d(dst + kHalfBytes, &tmA, 64, rowA, &full[st]);
        tc::tma_load_2d(dst + kABytes, &tmDK, 0, rowK, &full[st]);
        tc::tma_load_2d(dst + kABytes + kDKBytes / 2, &tmDK, 64, rowK, &full[st]);
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
      for (int s = 0;; ++s) {
        const int st = s % kStages;
        if (!tc::mbar_wait(&full[st], (s / kStages) & 1, abort_s)) break;
        const StepInfo e = info[st];
        if (e.j < 0) break;
        tc::tc_fence_after();
        const uint32_t a_base = tc::smem_u32(ring + st * kStageBytes);
        const uint32_t k_base = a_base + kABytes;
        bool ok = true;
        for (int k = 0; k < 2; ++k) {
          if (!((e.flags >> k) & 1)) continue;
          if (!tc::mbar_wait(&op_ready[k], e.p[k] & 1, abort_s)) {
            ok = false;
            break;
          }
          tc::tc_fence_after();
          const uint32_t d_t = tbase + 128u * k;
          const uint32_t a_t = tbase + 256u + kOpCols * k;
          const bool first = (e.flags >> (2 + k)) & 1;
          if (!first) {
            const uint32_t acc0 = e.g[k] < 1.0f ? 1u : 0u;
#pragma unroll
            for (int ks = 0; ks < kD / 16; ++ks)
              tc::mma_ts(d_t, a_t + 8u * ks, tc::sdesc_sw128(a_base + ks * 2048, kHalfBytes, 1024), kIdesc,
                         ks > 0 ? 1u : acc0);
          }
#pragma unroll
          for (int ks = 0; ks < kC / 16; ++ks)
            tc::mma_ts(d_t, a_t + 64u + 8u * ks, tc::sdesc_sw128(k_base + ks * 2048, kDKBytes / 2, 1024), kIdesc,
                       (first && ks == 0) ? 0u : 1u);
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
    // ------------- epilogue: group k (8 warps, 256 threads, named barrier 1 + k) -------------
    const int k = (warp - 2) >> 3;
    const int bar_id = 1 + k;
    const int q = warp & 3;
    const int h = ((warp - 2) & 7) >> 2;
    const int v = 32 * q + lane;
    const int col0 = 64 * h;
    const uint32_t lane_off = (uint32_t)(32 * q) << 16;
    const uint32_t d_addr0 = tbase + lane_off + 128u * k + col0;
    const uint32_t op_addr = tbase + lane_off + 256u + kOpCols * k;
    const int chain = k ? chains[1] : chains[0];
    const int cnt = chain >= 0 ? a.act_cnt[(long)bh * a.N + chain] : 0;
    __nv_bfloat16* out_row =
        chain >= 0 ? a.S_in + ((long)bh * a.N + chain) * kD * kD + (long)v * kD + col0 : nullptr;
    // c2 Ub_j^T row v, this thread's 32 of the C columns, into the operand
    auto put_ut = [&](int jn, float c2) {
      const uint4* src = (const uint4*)(a.UT + (((long)bh * a.N + jn) * kD + v) * kC + 32 * h);
      uint32_t w[16];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 u = src[i];
        const uint32_t uu[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = tc::mul2(make_float2(c2, c2), tc::bf16x2_to_float2(uu[e]));
          w[4 * i + e] = tc::pack_bf16x2(f.x, f.y);
        }
      }
      tc::tmem_st16(op_addr + 64u + 16u * h, w);
    };
    if (chain >= 0 && cnt == 0) {
      // a chain with nothing active has S_in = 0
      for (int e = 0; e < 8; ++e) ((uint4*)out_row)[e] = make_uint4(0u, 0u, 0u, 0u);
    } else if (chain >= 0) {
      // operand of the first step: Ub^T of its chunk (the state is zero)
      put_ut(a.act_idx[((long)bh * a.N + chain) * a.N], 1.0f);
      tc::tmem_wait_st();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&op_ready[k]);
    }
    float rho = 1.0f;
    for (int s = 0;; ++s) {
      const int st = s % kStages;
      const bool w = tc::mbar_wait(&full[st], (s / kStages) & 1, abort_s);
      const int jv = w ? ((volatile StepInfo*)info)[st].j : 0;
      // one vote per step: stop at the end marker or on a timeout anywhere
      if (tc::bar_any(bar_id, 256, !w || *abort_s != 0 || jv < 0)) break;
      const StepInfo e = info[st];
      const bool act = (e.flags >> k) & 1;
      const bool last = (e.flags >> (4 + k)) & 1;
      if (act) {
        const bool first = (e.flags >> (2 + k)) & 1;
        const float g = k ? e.g[1] : e.g[0];
        const float gn = k ? e.gn[1] : e.gn[0];
        const int jn = k ? e.jn[1] : e.jn[0];
        const int pk = k ? e.p[1] : e.p[0];
        tc::mbar_wait(&mma_done[k], pk & 1, abort_s);
        tc::tc_fence_after();
        rho = first ? g : (g < 1.0f ? rho * (1.0f - g) : rho);
        if (last) {
#pragma unroll
          for (int cc = 0; cc < 64; cc += 32) {
            uint32_t d[32];
            tc::tmem_ld32(d_addr0 + cc, d);
            tc::tmem_wait_ld();
            uint4* out = (uint4*)(out_row + cc);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              uint32_t o[4];
#pragma unroll
              for (int e2 = 0; e2 < 4; ++e2) {
                const float2 f = tc::mul2(make_float2(rho, rho), make_float2(__uint_as_float(d[8 * i + 2 * e2]),
                                                                             __uint_as_float(d[8 * i + 2 * e2 + 1])));
                o[e2] = tc::pack_bf16x2(f.x, f.y);
              }
              out[i] = make_uint4(o[0], o[1], o[2], o[3]);
            }
          }
        } else {
          const bool renorm = rho < 9.313225746e-10f;  // 2^-30
          const float scale = renorm ? rho : 1.0f;
          if (renorm) rho = 1.0f;
          const float c1 = gn < 1.0f ? gn / (1.0f - gn) : 1.0f;
          const float c2 = c1 / rho;
          const float2 c12 = make_float2(c1, c1), sc2 = make_float2(scale, scale);
#pragma unroll
          for (int cc = 0; cc < 64; cc += 32) {
            uint32_t d[32];
            tc::tmem_ld32(d_addr0 + cc, d);
            tc::tmem_wait_ld();
            uint32_t op[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              float2 x = make_float2(__uint_as_float(d[2 * i]), __uint_as_float(d[2 * i + 1]));
              if (renorm) {
                x = tc::mul2(sc2, x);
                d[2 * i] = __float_as_uint(x.x);
                d[2 * i + 1] = __float_as_uint(x.y);
              }
              const float2 o = tc::mul2(c12, x);
              op[i] = tc::pack_bf16x2(o.x, o.y);
            }
            if (renorm) tc::tmem_st32(d_addr0 + cc, d);
            tc::tmem_st16(op_addr + (col0 + cc) / 2, op);
          }
          put_ut(jn, c2);
        }
        tc::tmem_wait_st();
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
  const long rowsA = (long)c.B * c.H * c.ab_chunk_stride * kD;
  const long rowsK = (long)c.B * c.H * c.N * kC;
  CUtensorMap tmA, tmDK;
  cudaError_t e = make_tmap_rows128(&tmA, c.A, rowsA);
  if (e != cudaSuccess) return e;
  e = make_tmap_2d(&tmDK, c.DK, kD, rowsK, kD * 2, 64, 64);
  if (e != cudaSuccess) return e;
  ComposeTcArgs a;
  a.BH = c.B * c.H;
  a.N = c.N;
  a.ab_chunk_stride = c.ab_chunk_stride;
  a.act_idx = c.act_idx;
  a.act_g = c.act_g;
  a.act_cnt = c.act_cnt;
  a.UT = (const __nv_bfloat16*)c.UT;
  a.S_in = (__nv_bfloat16*)c.S_in;
  const size_t smem = 1024 + kStages * kStageBytes + 512;
  e = cudaFuncSetAttribute(compose_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int pairs = (c.N + 1) / 2;
  compose_tc_kernel<<<pairs * a.BH, kThreads, smem, s>>>(tmA, tmDK, a);
  return cudaGetLastError();
}

}  // namespace hla
