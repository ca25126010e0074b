// Internal launch interfaces between hla_api.cu and the kernel translation units.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace hla {

// Window representatives: at most this many per chunk (C / pool_window).
constexpr int kMaxWindows = 16;

struct GatesArgs {
  int B, H, N, d, mode;
  int win;                  // key representatives per chunk with windows (0: one pool per chunk)
  float c_d, bias, thr;
  const float* rq;          // [B,H,N,d]
  const float* rk;          // [B,H,N,d], or [B,H,N*win,d] with windows
  const float* user_gates;  // [B,H,N,N] (mode USER)
  int32_t* act_idx;         // [B,H,N,N] compacted ascending j
  float* act_g;             // [B,H,N,N] matching gates
  int32_t* act_cnt;         // [B,H,N]
  float* gates_out;         // optional [B,H,N,N]
  int32_t* active_idx_out;  // optional [B,H,N,N]
  int32_t* active_cnt_out;  // optional [B,H,N]
  bool pad_act_idx;         // pad act_idx rows beyond the count with -1
};

// Token-major input view of k/v/alpha/beta used by the transition kernels:
// element (b, h, t, c) of k is at k[b*sb + h*sh + t*st + c]; alpha at
// alpha[b*ab + h*ah + t*at].
struct TokenView {
  const void* k;
  const void* v;
  const float* alpha;
  const float* beta;
  long sb, sh, st;   // k/v strides (elements)
  long ab, ah, at;   // alpha/beta strides (elements)
  int alpha_vec;     // channel-wise decay: alpha (b, h, t, c) at b*ab + h*ah + t*at + c
                     // and beta (b, h, t) at (b*ab + h*ah + t*at) / d
};

struct TransArgs {
  int B, H, T, C, d, dtype;
  TokenView in;
  int n_chunks;          // chunks to process per (b,h) (complete + optional partial)
  void* A;               // [B,H,chunk_stride,d,d] (dtype) or null
  void* Bm;              // same
  long ab_chunk_stride;  // chunk stride of A/B (in chunks)
  long ab_chunk_offset;  // first chunk index written (decode close)
  float* Wb;             // [B,H,N,C,d] fp32 or null
  float* Ub;             // [B,H,N,C,d] fp32 or null
  float* ell;            // [B,H,N,C] fp32 or null
  const int32_t* close_m;   // decode close: per-b m_partial (before the step) or null
  const int32_t* close_n;   // decode close: per-b n_chunks or null
  // decode close into a factored cache: K, Wb, Ub ([.., chunk_stride, C, d]) and the
  // scales ([.., chunk_stride, C + 4]) of the closed chunk instead of A/B
  void* Kf;
  void* Wf;
  void* Uf;
  float* df;
};

// Prefill -> factored cache: the WY factors and scales of every complete chunk.
struct FactorFillArgs {
  int B, H, T, N, Nc, max_chunks;
  const void* k;       // [B,T,H,d] bf16 (input keys)
  const void* Wb;      // [B,H,N,C,d] bf16 (workspace)
  const void* Ub;
  const float* ell;    // [B,H,N,C]
  void* Kf;            // [B,H,max_chunks,C,d] bf16
  void* Wf;
  void* Uf;
  float* df;           // [B,H,max_chunks,C+4]
};

struct ComposeArgs {
  int B, H, N, d, dtype;
  const void* A;          // [B,H,ab_stride,d,d]
  const void* Bm;
  long ab_chunk_stride;
  const int32_t* act_idx; // [B,H,N,N]
  const float* act_g;
  const int32_t* act_cnt; // [B,H,N]
  float* S_in;            // [B,H,n_slots,d,d]: S_in(i) goes to slot i * slot_mult
  int slot_mult;          // 64-token sub-chunks per chunk (1 at C = 64)
  int n_slots;            // sub-chunks per (b,h)
  bool sparse;            // chunks may be skipped (threshold > 0)
  int32_t* order;         // [B,H,N] scratch for the pairing order (tensor-core path), or null
};

// Chunks of C = 64 s tokens (s > 1) are handled as s sub-chunks of 64 tokens.  The
// affine chains below connect the two levels (all matrices d x d, row-major):
//   merge    A_i = A_{is} A_{is+1} ... A_{is+s-1}
//            B_i = (...((B_{is} A_{is+1} + B_{is+1}) A_{is+2} + B_{is+2}) ...)
//            over the sub-chunk transitions of every complete chunk i;
//   advance  S_(i,k) = S_(i,k-1) A_{is+k-1} + B_{is+k-1}, S_(i,0) = S_in(i), the state
//            entering sub-chunk is+k, for every sub-chunk after the first of chunk i.
struct ChainArgs {
  int B, H, d, dtype;
  int s;                 // sub-chunks per chunk (2 or 4)
  const void* Asub;      // [B,H,sub_stride,d,d] (dtype): sub-chunk transitions
  const void* Bsub;
  long sub_stride;
  // merge
  int Nc;                // complete chunks per (b,h)
  void* Aout;            // [B,H,out_stride,d,d] (dtype)
  void* Bout;
  long out_stride;
  // advance
  int N, Nsub;           // chunks and sub-chunks per (b,h)
  void* S;               // [B,H,Nsub,d,d]: float32 (CUDA-core path) or bf16 (tensor-core path)
};

// Intra-chunk read-out by the token rule (channel-wise decay): every chunk runs the
// rule from its composed state S_in and emits o_t = S_t q_t.
struct ReadoutTokenArgs {
  int B, H, T, C, N, d, dtype;
  TokenView in;            // k, v, alpha (channel-wise), beta
  const void* q;           // [B,T,H,d], strides of in.k
  const void* S_in;        // [B,H,N,d,d] ([v][c]); bf16 if S_bf16 else float32
  bool S_bf16;
  void* o;                 // [B,T,H,d]
};

// Channel-wise decay on the tensor cores: per 64-token sub-chunk the decays folded
// into the keys and queries (chan_prep.cu).  Every operand is [B,H,Nsub,64,128] bf16
// (row t of sub-chunk n at ((b*H + h)*Nsub + n)*64 + t); gC is [B,H,Nsub,128] float32.
struct ChanPrepArgs {
  int B, H, T, Nsub;
  const void* k;        // [B,T,H,128] bf16
  const void* q;
  const float* alpha;   // [B,T,H,128]
  void* Kt;             // k o gamma_t
  void* Kh;             // k / gamma_t
  void* Kc;             // k o gamma_C / gamma_t
  void* Qt;             // q o gamma_t
  float* gC;            // gamma_C (the sub-chunk's whole decay per channel)
};

// Operands of the tensor-core transition / read-out kernels under channel-wise decay
// (null for the scalar decay).
struct ChanOperands {
  const void* Kt;
  const void* Kh;
  const void* Kc;
  const void* Qt;
  const float* gC;
};

struct ReadoutArgs {
  int B, H, T, C, N, d, dtype;
  const void* q;          // [B,T,H,d]
  const void* k;
  const float* S_in;      // [B,H,N,d,d]
  const float* Wb;        // [B,H,N,C,d]
  const float* Ub;
  const float* ell;       // [B,H,N,C]
  void* o;                // [B,T,H,d]
};

struct DecodeArgs {
  int B, H, C, d, dtype, mode, max_chunks;
  int win;             // window pools per closed chunk (0: one pool per chunk)
  int alpha_vec;       // channel-wise decay: alpha [B,H,d], buf_alpha [B,H,C,d]
  float tau, c_d, bias, thr;
  const void* q;   // [B,H,d]
  const void* k;
  const void* v;
  const float* alpha;  // [B,H]
  const float* beta;
  const void* q_route;
  const void* k_route;
  void* o;
  // cache
  const void* A;
  const void* Bm;
  int format;          // hla_cache_format
  void* Kf;            // factored: [B,H,max_chunks,C,d]
  void* Wf;
  void* Uf;
  float* df;           // factored: [B,H,max_chunks,C+4]
  float* rk;           // [B,H,max_chunks,max(win,1),d]
  void* buf_k;
  void* buf_v;
  void* buf_qr;
  void* buf_kr;
  float* buf_alpha;
  float* buf_beta;
  int32_t* n_chunks;
  int32_t* m_partial;
  // workspace
  int32_t* act_idx;  // [B,H,max_chunks]
  float* act_g;      // [B,H,max_chunks]
  int32_t* act_cnt;  // [B,H]: length of each active list (dense-cache streaming kernels)
};

cudaError_t launch_pools(const void* x0, const void* x1, float* r0, float* r1, int B, int T, int H, int d,
                         int C, int out_chunk_stride, float tau, int dtype, cudaStream_t s);
cudaError_t launch_gates(const GatesArgs& a, cudaStream_t s);
cudaError_t launch_transitions(const TransArgs& a, cudaStream_t s);
cudaError_t launch_compose(const ComposeArgs& a, cudaStream_t s);
cudaError_t launch_readout(const ReadoutArgs& a, cudaStream_t s);
cudaError_t launch_decode_main(const DecodeArgs& a, cudaStream_t s);
cudaError_t launch_decode_close(const DecodeArgs& a, cudaStream_t s);
cudaError_t launch_cache_fill(const DecodeArgs& c, const float* rk_ws, const void* q_route, const void* k_route,
                              const void* k, const void* v, const float* alpha, const float* beta, int T,
                              cudaStream_t s);
cudaError_t read_error_word_decode(unsigned int* out, bool clear);
cudaError_t read_error_word_compose_tc(unsigned int* out, bool clear);
cudaError_t launch_compose_tc(const ComposeArgs& a, bool scan, cudaStream_t s);
cudaError_t launch_decode_stream(const DecodeArgs& a, cudaStream_t s);
cudaError_t launch_transitions_tc(const TransArgs& t, cudaStream_t s, const ChanOperands* chan = nullptr);
cudaError_t launch_factor_fill(const FactorFillArgs& f, cudaStream_t s);
cudaError_t launch_decode_stream_factored(const DecodeArgs& a, cudaStream_t s);
cudaError_t launch_readout_tc(const ReadoutArgs& r, const void* S_in_bf16, const void* Wb_bf16, const void* Ub_bf16,
                              cudaStream_t s, const ChanOperands* chan = nullptr);
cudaError_t read_error_word_transitions_tc(unsigned int* out, bool clear);
cudaError_t read_error_word_readout_tc(unsigned int* out, bool clear);
cudaError_t read_error_word_decode_stream(unsigned int* out, bool clear);
cudaError_t read_error_word_wait_check(unsigned int* out, bool clear);
cudaError_t read_error_word_chain_tc(unsigned int* out, bool clear);
cudaError_t read_error_word_chan_prep(unsigned int* out, bool clear);
cudaError_t launch_chan_prep(const ChanPrepArgs& a, cudaStream_t s);
cudaError_t launch_chain_merge(const ChainArgs& a, cudaStream_t s);
cudaError_t launch_chain_advance(const ChainArgs& a, cudaStream_t s);
// Transitions of chunks of a.C > 64 tokens by the token rule itself (CUDA cores);
// same close_m / close_n semantics as launch_transitions.  Writes A/B only.
cudaError_t launch_transitions_token(const TransArgs& a, cudaStream_t s);
cudaError_t launch_readout_token(const ReadoutTokenArgs& a, cudaStream_t s);
cudaError_t launch_gate_support(const float* gates, int B, int H, int N, float thr, float* mass_out,
                                float* support_out, cudaStream_t s);
cudaError_t launch_wait_check(uint64_t limit_ns, bool complete, cudaStream_t s);

}  // namespace hla
