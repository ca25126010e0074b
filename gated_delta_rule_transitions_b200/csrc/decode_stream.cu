// Decode step for bf16 caches with d = 128: the active-chunk chain streams A_j and B_j
// from HBM through a TMA-fed shared-memory ring.
//
// HLA summary page, "Key Contributions" 3 (dynamic autoregressive decoding) and
// "Methodology in Plain English" paras. 3-4 (gated transitions; chunks below the
// threshold are skipped, so they are never read).  Same steps as the portable decode
// kernel: append the token, sweep the open chunk right to left (x = A_p q,
// y0 = B_p q), pool the open chunk's route queries, gate every closed chunk, then
//   for active j descending:  y += g_j B_j x;  x <- (1-g_j) x + g_j A_j x
// and o = y + y0.  The chain is bound by HBM: each active chunk costs 64 KiB of bf16
// and 4 d^2 flops.  One CTA per (sequence, head), two CTAs per SM: warps 0-3 compute
// (thread = row r), warp 4 issues TMA loads of A_j and B_j (128-byte swizzle, 64-column
// boxes) into a ring of three 32 KiB units, so about three chunks are in flight per SM.
//
// With routed gates and one key pool per chunk, the gate prologue reads every closed
// chunk's pool (512 B each; 256 KiB per (sequence, head) at 512 chunks -- as many
// bytes as four active chunks).  Those pools go through the same ring first: pieces
// of 64 pools (32 KiB, four 32-column boxes of float32 with the 128-byte swizzle),
// issued by the producer while the compute warps sweep the open chunk, so the
// pools stream from HBM as fast as the A_j/B_j tiles do.  Each pool is scored by one
// thread from shared memory (the swizzle keeps its 16-byte reads conflict-free).
#include <cstring>

#include "common.cuh"
#include "kernels.cuh"
#include "routing_recipe.cuh"
#include "tc_common.cuh"

namespace hla {

HLA_DEFINE_ERROR_WORD(decode_stream)

cudaError_t make_tmap_rows128(CUtensorMap* m, const void* base, long rows);
cudaError_t make_tmap_2d(CUtensorMap* m, const void* base, long inner, long rows, long row_stride_bytes,
                         int box_inner, int box_rows);

namespace {

typedef CUresult (*EncodeTiledFnF32)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                     const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                     CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// Float32 tensor map over `rows` rows of 128 values (the key pools of a cache), box
// 32 values (128 bytes) x box_rows rows, 128-byte swizzle.
cudaError_t make_tmap_pools(CUtensorMap* m, const float* base, long rows, int box_rows) {
  static EncodeTiledFnF32 fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFnF32)p;
  }
  if (fn == nullptr) return cudaErrorNotSupported;
  cuuint64_t dims[2] = {128, (cuuint64_t)rows};
  cuuint64_t strides[1] = {128 * 4};
  cuuint32_t box[2] = {32, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

constexpr int kD = 128;
constexpr int kHalf = kD * 64 * 2;       // 16 KiB: one 64-column box of a 128x128 bf16 matrix
constexpr int kCompute = 128;
constexpr int kThreads = kCompute + 32;

__device__ __forceinline__ float blk_sum(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  tc::bar_sync(1, kCompute);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  tc::bar_sync(1, kCompute);
  return red[0] + red[1] + red[2] + red[3];
}

// Steps shared by the streaming kernels, run by the kCompute threads (thread = channel):
// append the token to the open chunk, sweep the open chunk right to left (x = A_p q,
// y0 = B_p q), pool the open chunk's route queries, gate every closed chunk and write
// the ascending active list.  Returns the active count; x and y0 are this thread's.
// The flags leave steps to the caller: gates_here false -- the routed gates (rq is
// written); do_append / do_sweep / do_pool false -- the append, the sweep (x = y0 = 0)
// or the query pool.
__device__ __forceinline__ int decode_prologue(const DecodeArgs& a, int bh, int n, int m, float* rq, float* red,
                                             int* wcount, float& x, float& y0, bool gates_here = true,
                                             bool do_append = true, bool do_sweep = true, bool do_pool = true) {
  const int tid = threadIdx.x;
  const int C = a.C;
  const int mp = m + 1;
  int32_t* act_idx = a.act_idx + (long)bh * a.max_chunks;
  float* act_g = a.act_g + (long)bh * a.max_chunks;
  const long tok = (long)bh * kD + tid;
  const long bslot = ((long)bh * C + m) * kD + tid;
  if (do_append) {
    const __nv_bfloat16* qr_in = (const __nv_bfloat16*)(a.q_route ? a.q_route : a.q);
    const __nv_bfloat16* kr_in = (const __nv_bfloat16*)(a.k_route ? a.k_route : a.k);
    ((__nv_bfloat16*)a.buf_k)[bslot] = ((const __nv_bfloat16*)a.k)[tok];
    ((__nv_bfloat16*)a.buf_v)[bslot] = ((const __nv_bfloat16*)a.v)[tok];
    ((__nv_bfloat16*)a.buf_qr)[bslot] = qr_in[tok];
    ((__nv_bfloat16*)a.buf_kr)[bslot] = kr_in[tok];
    if (a.alpha_vec) a.buf_alpha[((long)bh * C + m) * kD + tid] = a.alpha[(long)bh * kD + tid];
    if (tid == 0) {
      if (!a.alpha_vec) a.buf_alpha[(long)bh * C + m] = a.alpha[bh];
      a.buf_beta[(long)bh * C + m] = a.beta[bh];
    }
    tc::bar_sync(1, kCompute);
    __threadfence_block();
  }
  const __nv_bfloat16* bk = (const __nv_bfloat16*)a.buf_k + (long)bh * C * kD;
  const __nv_bfloat16* bv = (const __nv_bfloat16*)a.buf_v + (long)bh * C * kD;
  // (1) open-chunk sweep
  x = do_sweep ? ldf((const __nv_bfloat16*)a.q + tok) : 0.0f;
  y0 = 0.0f;
  for (int t = do_sweep ? mp - 1 : -1; t >= 0; --t) {
    const float kt = ldf(bk + (long)t * kD + tid);
    const float c = blk_sum(kt * x, red);
    const float bt = a.buf_beta[(long)bh * C + t];
    // scalar decay, or this channel's decay
    const float at = a.alpha_vec ? a.buf_alpha[((long)bh * C + t) * kD + tid] : a.buf_alpha[(long)bh * C + t];
    y0 = fmaf(bt * c, ldf(bv + (long)t * kD + tid), y0);
    x = at * (x - bt * c * kt);
  }
  // (2) gates and the ascending active list
  int cnt = 0;
  if (a.mode != HLA_GATES_ZERO && n > 0 && (do_pool || gates_here)) {
    const route::Consts K = route::make_consts();
    if (a.mode == HLA_GATES_ROUTED && do_pool) {
      const __nv_bfloat16* bq = (const __nv_bfloat16*)a.buf_qr + (long)bh * C * kD + tid;
      const float inv_tau = __fdiv_rn(1.0f, a.tau);
      float mx = __fmul_rn(ldf(bq), inv_tau);
      for (int t = 1; t < mp; ++t) mx = fmaxf(mx, __fmul_rn(ldf(bq + (long)t * kD), inv_tau));
      float s = 0.0f;
      for (int t = 0; t < mp; ++t)
        s = __fadd_rn(s, route::rexp(route::pool_shift(ldf(bq + (long)t * kD), inv_tau, mx), K));
      rq[tid] = __fmul_rn(a.tau, __fadd_rn(mx, route::rlog(__fdiv_rn(s, (float)mp), K)));
      tc::bar_sync(1, kCompute);
    }
    if (!gates_here) return 0;
    const int W = a.win > 0 ? a.win : 1;
    const float* rk = a.rk + (long)bh * a.max_chunks * W * kD;
    for (int jb = 0; jb < n; jb += kCompute) {
      const int j = jb + tid;
      float g = 1.0f;
      bool keep = false;
      if (j < n) {
        if (a.mode == HLA_GATES_ROUTED && a.win > 0) {
          // log-sum-exp over the closed chunk's window representatives
          float t[kMaxWindows];
          const float m = route::window_scores(rq, rk + (long)j * W * kD, a.win, kD, a.c_d, t);
          g = route::gate_from_window_scores(t, a.win, m, a.bias, K);
        } else if (a.mode == HLA_GATES_ROUTED) {
          const float4* rkj = (const float4*)(rk + (long)j * kD);
          float dot = 0.0f;
          for (int c4 = 0; c4 < kD / 4; ++c4) {
            const float4 r4 = rkj[c4];
            dot = route::dot_step(dot, rq[4 * c4 + 0], r4.x);
            dot = route::dot_step(dot, rq[4 * c4 + 1], r4.y);
            dot = route::dot_step(dot, rq[4 * c4 + 2], r4.z);
            dot = route::dot_step(dot, rq[4 * c4 + 3], r4.w);
          }
          g = route::gate_from_dot(dot, a.c_d, a.bias, K);
        }
        keep = a.thr <= 0.0f || g >= a.thr;
      }
      const unsigned int bal = __ballot_sync(0xFFFFFFFFu, keep);
      const int w = tid >> 5;
      if ((tid & 31) == 0) wcount[w] = __popc(bal);
      tc::bar_sync(1, kCompute);
      int before = 0, total = 0;
#pragma unroll
      for (int k2 = 0; k2 < 4; ++k2) {
        if (k2 < w) before += wcount[k2];
        total += wcount[k2];
      }
      if (keep) {
        const int pos = cnt + before + __popc(bal & ((1u << (tid & 31)) - 1u));
        act_idx[pos] = j;
        act_g[pos] = g;
      }
      cnt += total;
      tc::bar_sync(1, kCompute);
    }
  }
  return cnt;
}

// Dense cache (bf16, d = 128): two kernels per decode step.
//
// decode_gates_kernel -- one CTA per (sequence, head), three CTAs per SM: appends the
// token to the open chunk, pools the open chunk's route queries, scores every closed
// chunk's key pool and writes the ascending active list and its length.  With routed
// gates and one pool per chunk the pools stream in by TMA in pieces of 64 pools
// (32 KiB, four 32-column boxes of float32 with the 128-byte swizzle) through a ring
// of two pieces; threads 0-63 score the first piece of a round and threads 64-127 the
// second (one fma chain over ascending channels per pool, the recipe's order; the
// swizzle keeps the 16-byte reads conflict-free).  Every (sequence, head) is gated at
// once across the GPU, and the 512 B per closed chunk stream at full bandwidth.
//
// decode_stream_kernel -- one CTA per (sequence, head), two CTAs per SM: the producer
// reads the list's length and streams the active chunks at once, j descending, two
// 32 KiB units each (a 64-column half of A_j with the same half of B_j) through a ring
// of three units, while the compute warps sweep the open chunk; then the chain, a unit
// handed back to the producer as soon as its pass is done.
constexpr int kUnit = 2 * kHalf;                    // 32 KiB
constexpr int kUnits = 3;
constexpr int kPoolRows = kUnit / (kD * 4);          // 64 key pools of 512 B per piece
constexpr int kGPieces = 2;                          // ring of the gate kernel

__global__ void __launch_bounds__(kThreads, 3)
    decode_gates_kernel(const __grid_constant__ CUtensorMap tmR, DecodeArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* ring = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* full = (uint64_t*)(ring + kGPieces * kUnit);
  uint64_t* empty = full + kGPieces;
  float* rq = (float*)(empty + kGPieces);    // [kD]
  float* red = rq + kD;                      // [4]
  int* wcount = (int*)(red + 4);             // [4]
  volatile int* abort_s = (volatile int*)(wcount + 4);

  const int bh = blockIdx.x;
  const int b = bh / a.H;
  const int tid = threadIdx.x;
  const int n = a.n_chunks[b];
  const int m = a.m_partial[b];
  int32_t* act_idx = a.act_idx + (long)bh * a.max_chunks;
  float* act_g = a.act_g + (long)bh * a.max_chunks;
  const bool stream_pools = a.mode == HLA_GATES_ROUTED && a.win == 0 && n > 0;
  const int npieces = stream_pools ? (n + kPoolRows - 1) / kPoolRows : 0;

  if (tid == 0) {
    for (int u = 0; u < kGPieces; ++u) {
      tc::mbar_init(&full[u], 1);
      tc::mbar_init(&empty[u], 1);
    }
    *abort_s = 0;
    tc::mbar_fence_init();
    tc::fence_async_smem();
  }
  __syncthreads();

  if (tid >= kCompute) {
    // ---------------- TMA producer (warp 4, lane 0): the key pool pieces ----------------
    if (tid == kCompute && npieces > 0) {
      tc::tma_prefetch_desc(&tmR);
      int u = 0;
      for (; u < npieces; ++u) {
        const int st = u % kGPieces;
        if (u >= kGPieces && !tc::mbar_wait(&empty[st], ((u / kGPieces) - 1) & 1, abort_s)) break;
        const int row = (int)((long)bh * a.max_chunks + (long)u * kPoolRows);
        tc::mbar_arrive_expect_tx(&full[st], kUnit);
        uint8_t* dst = ring + st * kUnit;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) tc::tma_load_2d(dst + q4 * (kUnit / 4), &tmR, 32 * q4, row, &full[st]);
      }
      if (*abort_s)
        for (int t = max(0, u - kGPieces); t < u; ++t)
          tc::mbar_wait(&full[t % kGPieces], (t / kGPieces) & 1, nullptr, 200000000ull);
    }
    __syncwarp();
  } else {
    // ---------------- compute (warps 0-3), thread = channel ----------------
    float x, y0;
    // append, query pool, and (without streamed pools) the gates
    int cnt = decode_prologue(a, bh, n, m, rq, red, wcount, x, y0, !stream_pools, true, false, true);
    bool ok = true;
    if (stream_pools) {
      const route::Consts K = route::make_consts();
      const int half = tid >> 6, r = tid & 63;
      int u = 0;
      for (int pc0 = 0; pc0 < npieces; pc0 += 2) {
        const bool two = pc0 + 1 < npieces;
        bool got = tc::mbar_wait(&full[u % kGPieces], (u / kGPieces) & 1, abort_s);
        if (two) got = got && tc::mbar_wait(&full[(u + 1) % kGPieces], ((u + 1) / kGPieces) & 1, abort_s);
        ok = tc::bar_all(1, kCompute, got);
        if (!ok) break;
        const int mine = u + half;
        const int j = (pc0 + half) * kPoolRows + r;
        float dot = 0.0f;
        if (half == 0 || two) {
          const uint8_t* piece = ring + (mine % kGPieces) * kUnit;
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const uint8_t* rowp = piece + q4 * (kUnit / 4) + r * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const float4 r4 = *(const float4*)(rowp + ((c ^ (r & 7)) << 4));
              const int c0 = 32 * q4 + 4 * c;
              dot = route::dot_step(dot, rq[c0 + 0], r4.x);
              dot = route::dot_step(dot, rq[c0 + 1], r4.y);
              dot = route::dot_step(dot, rq[c0 + 2], r4.z);
              dot = route::dot_step(dot, rq[c0 + 3], r4.w);
            }
          }
        }
        float g = 0.0f;
        bool keep = false;
        if (j < n) {
          g = route::gate_from_dot(dot, a.c_d, a.bias, K);
          keep = a.thr <= 0.0f || g >= a.thr;
        }
        const unsigned int bal = __ballot_sync(0xFFFFFFFFu, keep);
        const int w = tid >> 5;
        if ((tid & 31) == 0) wcount[w] = __popc(bal);
        tc::bar_sync(1, kCompute);  // also: every thread has read this round's pieces
        if (tid == 0) {
          tc::mbar_arrive(&empty[u % kGPieces]);
          if (two) tc::mbar_arrive(&empty[(u + 1) % kGPieces]);
        }
        u += two ? 2 : 1;
        int before = 0, total = 0;
#pragma unroll
        for (int k2 = 0; k2 < 4; ++k2) {
          if (k2 < w) before += wcount[k2];
          total += wcount[k2];
        }
        if (keep) {
          const int pos = cnt + before + __popc(bal & ((1u << (tid & 31)) - 1u));
          act_idx[pos] = j;
          act_g[pos] = g;
        }
        cnt += total;
        tc::bar_sync(1, kCompute);
      }
    }
    if (tid == 0) a.act_cnt[bh] = ok ? cnt : 0;
  }
  __syncthreads();
  if (tid == 0 && *abort_s) report_device_error(kErrMbarTimeout);
  // the stream kernel, launched as this grid's programmatic dependent, may start its
  // CTAs now (it waits for this grid's completion before reading anything)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__global__ void __launch_bounds__(kThreads, 2)
    decode_stream_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                         DecodeArgs a) {
  // launched as the gate kernel's programmatic dependent: everything below reads its
  // results (or the step's appended token), so wait for that grid to complete first
  asm volatile("griddepcontrol.wait;" ::: "memory");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* ring = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* full = (uint64_t*)(ring + kUnits * kUnit);
  uint64_t* empty = full + kUnits;
  float* xs = (float*)(empty + kUnits);      // [2][kD]
  float* rq = xs + 2 * kD;                   // [kD] (not used: the gates are done)
  float* red = rq + kD;                      // [4]
  int* wcount = (int*)(red + 4);             // [4]
  volatile int* abort_s = (volatile int*)(wcount + 4);

  const int bh = blockIdx.x;
  const int b = bh / a.H;
  const int tid = threadIdx.x;
  const int n = a.n_chunks[b];
  const int m = a.m_partial[b];
  const int32_t* act_idx = a.act_idx + (long)bh * a.max_chunks;
  const float* act_g = a.act_g + (long)bh * a.max_chunks;
  const int cnt = a.act_cnt[bh];

  if (tid == 0) {
    for (int u = 0; u < kUnits; ++u) {
      tc::mbar_init(&full[u], 1);
      tc::mbar_init(&empty[u], 1);
    }
    *abort_s = 0;
    tc::mbar_fence_init();
    tc::fence_async_smem();
  }
  __syncthreads();

  if (tid >= kCompute) {
    // ---------------- TMA producer (warp 4, lane 0): two units per active chunk ----------------
    if (tid == kCompute && cnt > 0) {
      tc::tma_prefetch_desc(&tmA);
      tc::tma_prefetch_desc(&tmB);
      int u = 0;
      bool go = true;
      for (int p = cnt - 1; go && p >= 0; --p) {
        const int j = act_idx[p];
        const int row = (int)(((long)bh * a.max_chunks + j) * kD);
        for (int hh = 0; hh < 2; ++hh, ++u) {
          const int st = u % kUnits;
          if (u >= kUnits && !tc::mbar_wait(&empty[st], ((u / kUnits) - 1) & 1, abort_s)) {
            go = false;
            break;
          }
          tc::mbar_arrive_expect_tx(&full[st], kUnit);
          uint8_t* dst = ring + st * kUnit;
          tc::tma_load_2d(dst, &tmA, 64 * hh, row, &full[st]);
          tc::tma_load_2d(dst + kHalf, &tmB, 64 * hh, row, &full[st]);
        }
      }
      if (*abort_s)
        for (int t = max(0, u - kUnits); t < u; ++t)
          tc::mbar_wait(&full[t % kUnits], (t / kUnits) & 1, nullptr, 200000000ull);
    }
    __syncwarp();
  } else {
    // ---------------- compute (warps 0-3), thread = channel / row ----------------
    float x, y0;
    decode_prologue(a, bh, n, m, rq, red, wcount, x, y0, false, false, true, false);  // the sweep only
    const long tok = (long)bh * kD + tid;
    xs[tid] = x;
    tc::bar_sync(1, kCompute);
    // active chain, descending j: two units per chunk (column halves of A_j, B_j)
    float y = 0.0f;
    int cur = 0, u = 0;
    bool ok = true;
    for (int p = cnt - 1; ok && p >= 0; --p) {
      const float* xc = xs + cur * kD;
      float ax0 = 0.f, ax1 = 0.f, bx0 = 0.f, bx1 = 0.f;
      for (int hh = 0; hh < 2; ++hh, ++u) {
        const int st = u % kUnits;
        ok = tc::bar_all(1, kCompute, tc::mbar_wait(&full[st], (u / kUnits) & 1, abort_s));
        if (!ok) break;
        const uint8_t* stA = ring + st * kUnit;
        const uint8_t* stB = stA + kHalf;
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
          const int off = tid * 128 + ((c8 ^ (tid & 7)) << 4);
          const uint4 wa = *(const uint4*)(stA + off);
          const uint4 wb = *(const uint4*)(stB + off);
          const float4 x0 = *(const float4*)(xc + hh * 64 + c8 * 8);
          const float4 x1 = *(const float4*)(xc + hh * 64 + c8 * 8 + 4);
          ax0 = fmaf(tc::bf16lo(wa.x), x0.x, ax0);
          ax1 = fmaf(tc::bf16hi(wa.x), x0.y, ax1);
          ax0 = fmaf(tc::bf16lo(wa.y), x0.z, ax0);
          ax1 = fmaf(tc::bf16hi(wa.y), x0.w, ax1);
          ax0 = fmaf(tc::bf16lo(wa.z), x1.x, ax0);
          ax1 = fmaf(tc::bf16hi(wa.z), x1.y, ax1);
          ax0 = fmaf(tc::bf16lo(wa.w), x1.z, ax0);
          ax1 = fmaf(tc::bf16hi(wa.w), x1.w, ax1);
          bx0 = fmaf(tc::bf16lo(wb.x), x0.x, bx0);
          bx1 = fmaf(tc::bf16hi(wb.x), x0.y, bx1);
          bx0 = fmaf(tc::bf16lo(wb.y), x0.z, bx0);
          bx1 = fmaf(tc::bf16hi(wb.y), x0.w, bx1);
          bx0 = fmaf(tc::bf16lo(wb.z), x1.x, bx0);
          bx1 = fmaf(tc::bf16hi(wb.z), x1.y, bx1);
          bx0 = fmaf(tc::bf16lo(wb.w), x1.z, bx0);
          bx1 = fmaf(tc::bf16hi(wb.w), x1.w, bx1);
        }
        if (hh == 0) {
          // every thread has read this unit: hand it back to the producer
          tc::bar_sync(1, kCompute);
          if (tid == 0) tc::mbar_arrive(&empty[st]);
        } else {
          const float g = act_g[p];
          y = fmaf(g, bx0 + bx1, y);
          xs[(cur ^ 1) * kD + tid] = (1.0f - g) * xc[tid] + g * (ax0 + ax1);
          cur ^= 1;
          tc::bar_sync(1, kCompute);
          if (tid == 0) tc::mbar_arrive(&empty[st]);
        }
      }
    }
    stf((__nv_bfloat16*)a.o + tok, y + y0);
  }
  __syncthreads();
  if (tid == 0 && *abort_s) report_device_error(kErrMbarTimeout);
}

// ---------------------------------------------------------------------------------
// Factored cache.  A_j x = gamma_C x - Wb_j^T D_j (K_j x) and B_j x = Ub_j^T D_j (K_j x),
// so per active chunk the stage holds K_j, Wb_j, Ub_j (64 x 128 bf16 each, 128-byte
// swizzled 64-column boxes) and the scales (gamma_C / gamma_t, gamma_C): 48 KiB
// instead of 64 KiB.  Phase 1: z_t = K_j[t] . x on pairs of threads (t = tid / 2, one
// 64-column half each), z'_t = z_t gamma_C / gamma_t.  Phase 2: thread pairs own two
// columns and split the 64 rows between them (rows with bit 2 clear / set, so the two
// read disjoint banks): w = Wb^T z', u = Ub^T z'.  Then y += g u,
// x <- (1 - g + g gamma_C) x - g w.
constexpr int kFStages = 2;  // two CTAs per SM: 4 stages of 49 KiB in flight per SM
constexpr int kFTile = 64 * kD * 2;                 // 16 KiB: one 64 x 128 bf16 factor
constexpr int kFScale = (64 + 4) * 4;               // scales of one chunk
constexpr int kFStageBytes = 3 * kFTile + 1024;     // K, Wb, Ub, scales (1 KiB aligned)
constexpr uint32_t kFTx = 3 * kFTile + kFScale;

__global__ void __launch_bounds__(kThreads, 2)
    decode_stream_factored_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmW,
                                  const __grid_constant__ CUtensorMap tmU, DecodeArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* ring = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* full = (uint64_t*)(ring + kFStages * kFStageBytes);
  uint64_t* empty = full + kFStages;
  float* xs = (float*)(empty + kFStages);    // [2][kD]
  float* rq = xs + 2 * kD;                   // [kD]
  float* zs = rq + kD;                       // [64]
  float* red = zs + 64;                      // [4]
  int* wcount = (int*)(red + 4);             // [4]
  int* cnt_s = wcount + 4;                   // [1]
  volatile int* abort_s = (volatile int*)(cnt_s + 1);

  const int bh = blockIdx.x;
  const int b = bh / a.H;
  const int tid = threadIdx.x;
  const int n = a.n_chunks[b];
  const int m = a.m_partial[b];
  const int32_t* act_idx = a.act_idx + (long)bh * a.max_chunks;
  const float* act_g = a.act_g + (long)bh * a.max_chunks;

  if (tid == 0) {
    for (int s = 0; s < kFStages; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    *abort_s = 0;
    tc::mbar_fence_init();
    tc::fence_async_smem();
  }
  __syncthreads();

  if (tid >= kCompute) {
    // ---------------- TMA producer (warp 4, lane 0) ----------------
    tc::bar_sync(2, kThreads);
    if (tid == kCompute) {
      tc::tma_prefetch_desc(&tmK);
      tc::tma_prefetch_desc(&tmW);
      tc::tma_prefetch_desc(&tmU);
      const int cnt = *cnt_s;
      int s = 0;
      for (int p = cnt - 1; p >= 0; --p, ++s) {
        const int st = s % kFStages;
        if (s >= kFStages && !tc::mbar_wait(&empty[st], ((s / kFStages) - 1) & 1, abort_s)) break;
        const int j = act_idx[p];
        const long slot = (long)bh * a.max_chunks + j;
        const int row = (int)(slot * 64);
        tc::mbar_arrive_expect_tx(&full[st], kFTx);
        uint8_t* dst = ring + st * kFStageBytes;
        tc::tma_load_2d(dst, &tmK, 0, row, &full[st]);
        tc::tma_load_2d(dst + kFTile / 2, &tmK, 64, row, &full[st]);
        tc::tma_load_2d(dst + kFTile, &tmW, 0, row, &full[st]);
        tc::tma_load_2d(dst + kFTile + kFTile / 2, &tmW, 64, row, &full[st]);
        tc::tma_load_2d(dst + 2 * kFTile, &tmU, 0, row, &full[st]);
        tc::tma_load_2d(dst + 2 * kFTile + kFTile / 2, &tmU, 64, row, &full[st]);
        tc::bulk_load_1d(dst + 3 * kFTile, a.df + slot * (64 + 4), kFScale, &full[st]);
      }
      if (*abort_s)
        for (int t = max(0, s - kFStages); t < s; ++t)
          tc::mbar_wait(&full[t % kFStages], (t / kFStages) & 1, nullptr, 200000000ull);
    }
    __syncwarp();
  } else {
    // ---------------- compute (warps 0-3) ----------------
    float x, y0;
    const int cnt = decode_prologue(a, bh, n, m, rq, red, wcount, x, y0);
    const long tok = (long)bh * kD + tid;
    if (tid == 0) *cnt_s = cnt;
    xs[tid] = x;
    __threadfence_block();
    tc::bar_sync(2, kThreads);  // releases the producer
    const int pt = tid >> 1, ph = tid & 1;   // phase 1: row pt, column half ph
    const int cp = tid >> 1, th = tid & 1;   // phase 2: columns 2cp, 2cp+1; row set th
    const int cbox = (2 * cp) >> 6, c8 = ((2 * cp) & 63) >> 3, cw = ((2 * cp) & 7) * 2;
    float y = 0.0f;
    int cur = 0;
    bool ok = true;
    for (int p = cnt - 1, s = 0; p >= 0; --p, ++s) {
      const int st = s % kFStages;
      ok = tc::bar_all(1, kCompute, tc::mbar_wait(&full[st], (s / kFStages) & 1, abort_s));
      if (!ok) break;
      const uint8_t* stK = ring + st * kFStageBytes;
      const uint8_t* stW = stK + kFTile;
      const uint8_t* stU = stK + 2 * kFTile;
      const float* dfs = (const float*)(stK + 3 * kFTile);
      const float* xc = xs + cur * kD;
      // phase 1: z'_t
      {
        const uint8_t* krow = stK + ph * (kFTile / 2) + pt * 128;
        float z0 = 0.0f, z1 = 0.0f;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const uint4 w = *(const uint4*)(krow + ((q ^ (pt & 7)) << 4));
          const float4 x0 = *(const float4*)(xc + ph * 64 + q * 8);
          const float4 x1 = *(const float4*)(xc + ph * 64 + q * 8 + 4);
          z0 = fmaf(tc::bf16lo(w.x), x0.x, z0);
          z1 = fmaf(tc::bf16hi(w.x), x0.y, z1);
          z0 = fmaf(tc::bf16lo(w.y), x0.z, z0);
          z1 = fmaf(tc::bf16hi(w.y), x0.w, z1);
          z0 = fmaf(tc::bf16lo(w.z), x1.x, z0);
          z1 = fmaf(tc::bf16hi(w.z), x1.y, z1);
          z0 = fmaf(tc::bf16lo(w.w), x1.z, z0);
          z1 = fmaf(tc::bf16hi(w.w), x1.w, z1);
        }
        float z = z0 + z1;
        z += __shfl_xor_sync(0xFFFFFFFFu, z, 1);
        if (ph == 0) zs[pt] = z * dfs[pt];
      }
      tc::bar_sync(1, kCompute);
      // phase 2: w = Wb^T z', u = Ub^T z' for columns 2cp, 2cp+1 over this thread's rows
      float w0 = 0.0f, w1 = 0.0f, u0 = 0.0f, u1 = 0.0f;
#pragma unroll 8
      for (int k = 0; k < 32; ++k) {
        const int t = 8 * (k >> 2) + (k & 3) + 4 * th;
        const int off = cbox * (kFTile / 2) + t * 128 + ((c8 ^ (t & 7)) << 4) + cw;
        const uint32_t ww = *(const uint32_t*)(stW + off);
        const uint32_t uu = *(const uint32_t*)(stU + off);
        const float zt = zs[t];
        w0 = fmaf(tc::bf16lo(ww), zt, w0);
        w1 = fmaf(tc::bf16hi(ww), zt, w1);
        u0 = fmaf(tc::bf16lo(uu), zt, u0);
        u1 = fmaf(tc::bf16hi(uu), zt, u1);
      }
      w0 += __shfl_xor_sync(0xFFFFFFFFu, w0, 1);
      w1 += __shfl_xor_sync(0xFFFFFFFFu, w1, 1);
      u0 += __shfl_xor_sync(0xFFFFFFFFu, u0, 1);
      u1 += __shfl_xor_sync(0xFFFFFFFFu, u1, 1);
      // thread tid owns column tid = 2 cp + th
      const float wc = th ? w1 : w0, uc = th ? u1 : u0;
      const float g = act_g[p];
      const float rho = (1.0f - g) + g * dfs[64];
      y = fmaf(g, uc, y);
      xs[(cur ^ 1) * kD + tid] = rho * xc[tid] - g * wc;
      cur ^= 1;
      tc::bar_sync(1, kCompute);
      if (tid == 0) tc::mbar_arrive(&empty[st]);
    }
    stf((__nv_bfloat16*)a.o + tok, y + y0);
  }
  __syncthreads();
  if (tid == 0 && *abort_s) report_device_error(kErrMbarTimeout);
}

}  // namespace

cudaError_t launch_decode_stream_factored(const DecodeArgs& a, cudaStream_t s) {
  const long rows = (long)a.B * a.H * a.max_chunks * 64;
  CUtensorMap tmK, tmW, tmU;
  cudaError_t e = make_tmap_2d(&tmK, a.Kf, kD, rows, kD * 2, 64, 64);
  if (e == cudaSuccess) e = make_tmap_2d(&tmW, a.Wf, kD, rows, kD * 2, 64, 64);
  if (e == cudaSuccess) e = make_tmap_2d(&tmU, a.Uf, kD, rows, kD * 2, 64, 64);
  if (e != cudaSuccess) return e;
  const size_t smem = 1024 + kFStages * kFStageBytes + 2 * kFStages * 8 + (4 * kD + 64 + 16) * 4;
  e = cudaFuncSetAttribute(decode_stream_factored_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  decode_stream_factored_kernel<<<a.B * a.H, kThreads, smem, s>>>(tmK, tmW, tmU, a);
  return cudaGetLastError();
}

cudaError_t launch_decode_stream(const DecodeArgs& a, cudaStream_t s) {
  const long rows = (long)a.B * a.H * a.max_chunks * kD;
  CUtensorMap tmA, tmB;
  cudaError_t e = make_tmap_rows128(&tmA, a.A, rows);
  if (e != cudaSuccess) return e;
  e = make_tmap_rows128(&tmB, a.Bm, rows);
  if (e != cudaSuccess) return e;
  // key pools (one per chunk; with window representatives the gates read them directly)
  CUtensorMap tmR;
  std::memset(&tmR, 0, sizeof(tmR));
  if (a.mode == HLA_GATES_ROUTED && a.win == 0) {
    e = make_tmap_pools(&tmR, a.rk, (long)a.B * a.H * a.max_chunks, kPoolRows);
    if (e != cudaSuccess) return e;
  }
  const size_t gsmem = 1024 + kGPieces * kUnit + 2 * kGPieces * 8 + (kD + 16) * 4;
  e = cudaFuncSetAttribute(decode_gates_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gsmem);
  if (e != cudaSuccess) return e;
  decode_gates_kernel<<<a.B * a.H, kThreads, gsmem, s>>>(tmR, a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t smem = 1024 + kUnits * kUnit + 2 * kUnits * 8 + (4 * kD + 16) * 4;
  e = cudaFuncSetAttribute(decode_stream_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  // programmatic dependent launch: the stream CTAs are scheduled while the gate grid
  // drains and wait (griddepcontrol.wait) for it to complete
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.B * a.H);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, decode_stream_kernel, tmA, tmB, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace hla
