// Gated composition on the 5th-generation tensor cores (tcgen05 + TMEM + TMA),
// bf16 operands, float32 state.  d = 128, C = 64.
//
// HLA summary page, "Methodology in Plain English" paras. 3-4: for query chunk i,
//   S <- 0;  for j in active(i), ascending:  S <- S + g_ij ((S A_j + B_j) - S)
// and a chunk below the threshold is skipped (it is not in active(i)).
//
// One CTA runs two query chunks ("chains") of one head.  Per step j of the merged
// active lists, TMA brings A_j and B_j (bf16, 128-byte swizzle) into a 3-stage ring;
// for each chain active at j the MMA warp issues
//     D_k += Aop_k x A_j     (M = 128 rows v, N = 128 columns c, K = 128)
// where the float32 master state lives in tensor memory pre-scaled, D_k = (1-g) S,
// and the MMA operand Aop_k = bf16(g S) also lives in tensor memory.  The epilogue
// warps then add g B_j[v][c], giving S_new, and prepare the next active step of that
// chain: D_k <- (1 - g_next) S_new, Aop_k <- bf16(g_next S_new).  After a chain's
// last active step S_new is written to S_in (bf16, [v][c]).
//
// Warp roles: warp 0 TMA producer, warp 1 TMEM allocator + MMA issuer, warps 2-17
// epilogue (lane quarter = warp % 4, column quarter = (warp - 2) / 4).  The epilogue
// warps finish each step chain by chain, so one chain's epilogue overlaps the other
// chain's MMA.  Elementwise math uses packed float32 pairs.  All waits are bounded
// (about 2 s, then a device error word is set and the CTA exits cleanly).
//
// Scan mode (every gate one, the native-GDN reduction): S_in(j+1) = S_in(j) A_j + B_j,
// so one chain per head walks j = 0 .. N-2 once and stores every intermediate state;
// the work is N-1 steps per head instead of N(N-1)/2.
#include "common.cuh"
#include "kernels.cuh"
#include "tc_common.cuh"

namespace hla {

HLA_DEFINE_ERROR_WORD(compose_tc)

namespace {

constexpr int kD = 128;
constexpr int kStages = 3;
constexpr int kStageBytes = 2 * kD * kD * 2;     // A_j + B_j, bf16
constexpr int kHalfBytes = kD * 64 * 2;          // one 64-column box
constexpr int kThreads = 576;  // producer, MMA, 2 x 8 epilogue warps
constexpr uint32_t kIdesc = tc::idesc_bf16_f32(128, 128, /*a_mn=*/0, /*b_mn=*/1);

struct ComposeTcArgs {
  int BH, N;
  int head_major;
  const int32_t* order;  // [BH, N] query chunks in pairing order, or null (descending)
  long ab_chunk_stride;
  const int32_t* act_idx;
  const float* act_g;
  const int32_t* act_cnt;
  __nv_bfloat16* S_in;  // [B,H,n_slots,d,d] bf16, row v, column c; S_in(i) in slot i * slot_mult
  int slot_mult, n_slots;
};

#ifndef HLA_COMPOSE_LIST_PREFETCH
#define HLA_COMPOSE_LIST_PREFETCH 1
#endif
constexpr bool kListPrefetch = HLA_COMPOSE_LIST_PREFETCH != 0;

__device__ __forceinline__ void prefetch_l1(const void* p) {
  asm volatile("prefetch.global.L1 [%0];" ::"l"(p));
}

// Walks the merged ascending active lists of the two chains.  The list entries are
// read one step at a time by one thread; with kListPrefetch the lines 32 entries
// ahead are requested into L1 as the walk goes, so that each step's reads hit L1.
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
  bool last[2];

  __device__ void init(const ComposeTcArgs& a, int bh, const int i[2]) {
    for (int k = 0; k < 2; ++k) {
      p[k] = 0;
      if (i[k] >= 0) {
        const long row = (long)bh * a.N + i[k];
        idx[k] = a.act_idx + row * a.N;
        g[k] = a.act_g + row * a.N;
        cnt[k] = a.act_cnt[row];
        if (kListPrefetch) {
          // the first two lines of each list (entries 0-63 that exist)
          prefetch_l1(idx[k]);
          prefetch_l1(g[k]);
          if (cnt[k] > 32) {
            prefetch_l1(idx[k] + 32);
            prefetch_l1(g[k] + 32);
          }
        }
      } else {
        idx[k] = nullptr;
        g[k] = nullptr;
        cnt[k] = 0;
      }
    }
  }
  // Loads the next step; false when both lists are exhausted.
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
    }
    return true;
  }
  __device__ void advance() {
    for (int k = 0; k < 2; ++k)
      if (act[k]) {
        ++p[k];
        // one 128-byte line holds 32 entries: entering a line, ask for the one after it
        if (kListPrefetch && (p[k] & 31) == 0 && p[k] + 32 < cnt[k]) {
          prefetch_l1(idx[k] + p[k] + 32);
          prefetch_l1(g[k] + p[k] + 32);
        }
      }
  }
};

// One step of the merged schedule, published by the producer next to its stage.
struct StepInfo {
  int j;       // chunk index; -1 ends the schedule
  int flags;   // bit k: chain k active; bit 2+k: first step of chain k; bit 4+k: last step
  int p[2];    // index of this step in each chain's active list
  float g[2];  // gates at this step
  float gn[2]; // gates at each chain's next active step (0 if none)
};

// Pairing order for the composition when chunks may be skipped.  Per (b, h) the query
// chunks are sorted by their first active chunk, then the longer active list first,
// then the later chunk first; consecutive entries are paired into one CTA.  Chunks
// whose lists start at the same chunk share most of their active chunks, so one
// A_j/B_j tile in the ring serves both chains.  Bitonic sort of 64-bit keys in
// shared memory, P = power of two >= N <= 4096.
__global__ void __launch_bounds__(1024) chain_order_kernel(const int32_t* __restrict__ act_idx,
                                                           const int32_t* __restrict__ act_cnt, int N, int P,
                                                           int32_t* __restrict__ order) {
  extern __shared__ unsigned long long keys[];
  const int bh = blockIdx.x;
  for (int i = threadIdx.x; i < P; i += blockDim.x) {
    unsigned long long k = ~0ull;
    if (i < N) {
      const long row = (long)bh * N + i;
      const int cnt = act_cnt[row];
      const int first = cnt > 0 ? act_idx[row * N] : N;
      k = ((unsigned long long)first << 40) | ((unsigned long long)(N - cnt) << 20) | (unsigned long long)(N - 1 - i);
    }
    keys[i] = k;
  }
  __syncthreads();
  for (int size = 2; size <= P; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int t = threadIdx.x; t < P / 2; t += blockDim.x) {
        const int lo = 2 * stride * (t / stride) + (t % stride);
        const int hi = lo + stride;
        const bool up = (lo & size) == 0;
        const unsigned long long x = keys[lo], y = keys[hi];
        if ((x > y) == up) {
          keys[lo] = y;
          keys[hi] = x;
        }
      }
      __syncthreads();
    }
  }
  for (int i = threadIdx.x; i < N; i += blockDim.x) order[(long)bh * N + i] = N - 1 - (int)(keys[i] & 0xFFFFFu);
}

template <bool kScan>
__global__ void __launch_bounds__(kThreads, 1)
    compose_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      ComposeTcArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* ring = smem;  // kStages x [A half0 | A half1 | B half0 | B half1]
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
  // Grid order.  Head-major (with skipping: short chains whose time is the A_j/B_j
  // reads): the CTAs resident at one time share one head's A_j/B_j through L2.
  // Interleaved heads (dense: long chains): the longest chains of every head go first.
  const int npairs = (a.N + 1) / 2;
  const int pair = kScan ? 0 : (a.head_major ? blockIdx.x % npairs : blockIdx.x / a.BH);
  const int bh = kScan ? blockIdx.x : (a.head_major ? blockIdx.x / npairs : blockIdx.x % a.BH);
  // scan mode: chain 0 is the head's running state (its S_in rows move with j), chain 1 idles
  int chains[2];
  if (kScan) {
    chains[0] = 0;
    chains[1] = -1;
  } else if (a.order != nullptr) {
    // query chunks paired by the order kernel (shared active lists)
    const int32_t* o = a.order + (long)bh * a.N;
    chains[0] = o[2 * pair];
    chains[1] = 2 * pair + 1 < a.N ? o[2 * pair + 1] : -1;
  } else {
    chains[0] = a.N - 1 - 2 * pair;
    chains[1] = a.N - 2 - 2 * pair;
  }

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1 + 16);  // MMA commit + lane 0 of every epilogue warp
    }
    for (int k = 0; k < 2; ++k) {
      tc::mbar_init(&mma_done[k], 1);
      tc::mbar_init(&op_ready[k], 16);  // lane 0 of every epilogue warp
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

  if (warp == 0) {
    // ---------------- TMA producer (lane 0): walks the merged lists ----------------
    if (lane == 0) {
      Sched sc;
      if (!kScan) sc.init(a, bh, chains);
      int s = 0;
      bool ok = true;
      while (kScan ? s < a.N - 1 : sc.next()) {
        const int st = s % kStages;
        if (s >= kStages && !tc::mbar_wait(&empty[st], ((s / kStages) - 1) & 1, abort_s)) {
          ok = false;
          break;
        }
        StepInfo e;
        if (kScan) {
          sc.j = s;
          e.j = s;
          e.flags = 1 | ((s == 0) ? 4 : 0) | ((s == a.N - 2) ? 16 : 0);
          e.p[0] = s;
          e.p[1] = 0;
          e.g[0] = 1.0f;
          e.g[1] = 0.0f;
          e.gn[0] = (s == a.N - 2) ? 0.0f : 1.0f;
          e.gn[1] = 0.0f;
        } else {
          e.j = sc.j;
          e.flags = 0;
          for (int k = 0; k < 2; ++k) {
            e.flags |= (sc.act[k] ? 1 : 0) << k;
            e.flags |= (sc.first[k] ? 1 : 0) << (2 + k);
            e.flags |= (sc.last[k] ? 1 : 0) << (4 + k);
            e.p[k] = sc.p[k];
            e.g[k] = sc.gate[k];
            e.gn[k] = sc.gnext[k];
          }
        }
        info[st] = e;
        tc::mbar_arrive_expect_tx(&full[st], kStageBytes);  // releases info[st]
        const int row = (int)(((long)bh * a.ab_chunk_stride + sc.j) * kD);
        uint8_t* dst = ring + st * kStageBytes;
        tc::tma_load_2d(dst, &tmA, 0, row, &full[st]);
        tc::tma_load_2d(dst + kHalfBytes, &tmA, 64, row, &full[st]);
        tc::tma_load_2d(dst + 2 * kHalfBytes, &tmB, 0, row, &full[st]);
        tc::tma_load_2d(dst + 3 * kHalfBytes, &tmB, 64, row, &full[st]);
        if (!kScan) sc.advance();
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
        const uint32_t b_base = tc::smem_u32(ring + st * kStageBytes);
        bool ok = true;
        for (int k = 0; k < 2; ++k) {
          if (!((e.flags >> k) & 1) || ((e.flags >> (2 + k)) & 1)) continue;
          if (!tc::mbar_wait(&op_ready[k], (e.p[k] - 1) & 1, abort_s)) {
            ok = false;
            break;
          }
          tc::tc_fence_after();
          const uint32_t d_t = tbase + 128u * k;
          const uint32_t a_t = tbase + 256u + 64u * k;
#pragma unroll
          for (int ks = 0; ks < kD / 16; ++ks) {
            const uint64_t bd = tc::sdesc_sw128(b_base + ks * 2048, kHalfBytes, 1024);
            tc::mma_ts(d_t, a_t + 8u * ks, bd, kIdesc, (kScan && ks == 0) ? 0u : 1u);
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
    // ------------- epilogue: all 16 warps (512 threads, named barrier 1) -------------
    // Each step is finished chain by chain by every epilogue warp: warp w owns TMEM
    // lane quarter q = w % 4 (rows v = 32 q + lane) and the column quarter
    // [32 c4, 32 c4 + 32).  While the warps finish one chain, the tensor pipe runs the
    // other chain's MMA.
    const int q = warp & 3;
    const int c4 = (warp - 2) >> 2;
    const int v = 32 * q + lane;
    const int col0 = 32 * c4;
    const uint32_t lane_off = (uint32_t)(32 * q) << 16;
    __nv_bfloat16* out_row[2];
    for (int k = 0; k < 2; ++k) {
      const int chain = chains[k];
      out_row[k] = chain >= 0 ? a.S_in + ((long)bh * a.n_slots + (long)chain * a.slot_mult) * kD * kD +
                                    (long)v * kD + col0
                              : nullptr;
      // a chain with nothing active has S_in = 0 (in scan mode: S_in(0))
      if (chain >= 0 && (kScan || a.act_cnt[(long)bh * a.N + chain] == 0))
        for (int e = 0; e < 4; ++e) ((uint4*)out_row[k])[e] = make_uint4(0u, 0u, 0u, 0u);
    }
    for (int s = 0;; ++s) {
      const int st = s % kStages;
      const bool w = tc::mbar_wait(&full[st], (s / kStages) & 1, abort_s);
      const int jv = w ? ((volatile StepInfo*)info)[st].j : 0;
      // one vote per step: stop at the end marker or on a timeout anywhere
      if (tc::bar_any(1, 512, !w || *abort_s != 0 || jv < 0)) break;
      const StepInfo e = info[st];
      // B_j[v][col0 .. col0+32) from the swizzled box (half col0 / 64, 16-byte chunks)
      const uint8_t* brow = ring + st * kStageBytes + 2 * kHalfBytes + (col0 >> 6) * kHalfBytes + v * 128;
      uint32_t bw[16];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int c8 = ((col0 & 63) >> 3) + c;
        const uint4 w4 = *(const uint4*)(brow + ((c8 ^ (v & 7)) << 4));
        bw[4 * c + 0] = w4.x;
        bw[4 * c + 1] = w4.y;
        bw[4 * c + 2] = w4.z;
        bw[4 * c + 3] = w4.w;
      }
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        if (!((e.flags >> k) & 1)) continue;
        const bool first = (e.flags >> (2 + k)) & 1;
        const bool last = (e.flags >> (4 + k)) & 1;
        const float g = k ? e.g[1] : e.g[0];
        const float gn = k ? e.gn[1] : e.gn[0];
        const int pk = k ? e.p[1] : e.p[0];
        const uint32_t d_addr = tbase + lane_off + 128u * k + col0;
        uint32_t d[32];
        if (!first) {
          tc::mbar_wait(&mma_done[k], (pk - 1) & 1, abort_s);
          tc::tc_fence_after();
          tc::tmem_ld32(d_addr, d);
          tc::tmem_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) d[i] = 0u;
        }
        const float2 g2 = make_float2(g, g);
        if (kScan || last) {
          // the state after this step (scan mode: S_in(j + 1); else the chain's S_in)
          uint4* out = (uint4*)(out_row[k] + (kScan ? (long)(e.j + 1) * a.slot_mult * kD * kD : 0));
          uint32_t op[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float2 x = tc::fma2(g2, tc::bf16x2_to_float2(bw[i]),
                                      make_float2(__uint_as_float(d[2 * i]), __uint_as_float(d[2 * i + 1])));
            op[i] = tc::pack_bf16x2(x.x, x.y);
          }
#pragma unroll
          for (int i = 0; i < 4; ++i) out[i] = make_uint4(op[4 * i], op[4 * i + 1], op[4 * i + 2], op[4 * i + 3]);
          // scan mode: the same bf16(S) is the next operand; the next product starts from zero
          if (kScan && !last) tc::tmem_st16(tbase + lane_off + 256u + 64u * k + col0 / 2, op);
        } else {
          const float keep = 1.0f - gn;
          const float2 gn2 = make_float2(gn, gn), keep2 = make_float2(keep, keep);
          uint32_t op[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float2 x = tc::fma2(g2, tc::bf16x2_to_float2(bw[i]),
                                      make_float2(__uint_as_float(d[2 * i]), __uint_as_float(d[2 * i + 1])));
            const float2 o = tc::mul2(gn2, x);
            const float2 nn = tc::mul2(keep2, x);
            op[i] = tc::pack_bf16x2(o.x, o.y);
            d[2 * i] = __float_as_uint(nn.x);
            d[2 * i + 1] = __float_as_uint(nn.y);
          }
          tc::tmem_st32(d_addr, d);
          tc::tmem_st16(tbase + lane_off + 256u + 64u * k + col0 / 2, op);
        }
        tc::tmem_wait_st();
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0 && !last) tc::mbar_arrive(&op_ready[k]);
      }
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&empty[st]);
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

cudaError_t launch_compose_tc(const ComposeArgs& c, bool scan, cudaStream_t s) {
  if (c.N <= 0) return cudaSuccess;
  if (c.ab_chunk_stride <= 0)  // no complete chunk: every composed state is zero
    return cudaMemsetAsync(c.S_in, 0, (size_t)c.B * c.H * c.n_slots * kD * kD * sizeof(__nv_bfloat16), s);
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
  a.slot_mult = c.slot_mult;
  a.n_slots = c.n_slots;
  a.head_major = c.sparse ? 1 : 0;
  a.order = nullptr;
  if (!scan && c.sparse && c.order != nullptr && c.N <= 4096) {
    int P = 1;
    while (P < c.N) P <<= 1;
    const size_t osmem = (size_t)P * sizeof(unsigned long long);
    e = cudaFuncSetAttribute(chain_order_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)osmem);
    if (e != cudaSuccess) return e;
    chain_order_kernel<<<a.BH, 1024, osmem, s>>>(c.act_idx, c.act_cnt, c.N, P, c.order);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    a.order = c.order;
  }
  const size_t smem = 1024 + kStages * kStageBytes + 512;
  if (scan) {
    e = cudaFuncSetAttribute(compose_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    compose_tc_kernel<true><<<a.BH, kThreads, smem, s>>>(tmA, tmB, a);
    return cudaGetLastError();
  }
  e = cudaFuncSetAttribute(compose_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int pairs = (c.N + 1) / 2;
  compose_tc_kernel<false><<<pairs * a.BH, kThreads, smem, s>>>(tmA, tmB, a);
  return cudaGetLastError();
}

}  // namespace hla
