/*
 * hla.h -- C ABI of libhla.so: Hybrid Linear Attention (HLA) over Gated DeltaNet,
 * prefill and decode hot path on one NVIDIA B200 (sm_100a).
 *
 * Source passages (HLA: Expressive Hybrid Linear Attention via Chunk-Wise Dynamic
 * Mixing, ai.info AI summary page):
 *   - "Methodology in Plain English", para. 1: per-token affine rule of Gated
 *     DeltaNet; a whole chunk is summarised exactly by one (matrix, additive term)
 *     pair because affine maps compose.
 *   - same section, para. 2: each chunk gets a pooled representative; a query's
 *     score against it is squashed through a sigmoid into a weight in (0, 1).
 *   - same section, para. 3: the weight interpolates the chunk's full transition
 *     with the identity; the current chunk has weight one; future chunks are masked.
 *   - same section, para. 4: weights below an inference threshold are set to zero
 *     without renormalisation, which makes skipping that chunk exact.
 *   - "Key Contributions" 3: training/prefill and dynamic autoregressive decoding.
 *   - "Overview": log-mean-exp pooled routing gates.
 *
 * Definitions used throughout (per sequence b and head h; d_k = d_v = d):
 *   token rule   S_t = S_{t-1} alpha_t (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
 *                o_t = S_t q_t            (S is d_v x d_k; no scaling of q)
 *   chunk c      tokens cC .. cC+C-1 act as S -> S A_c + B_c (exact)
 *   pools        r_c = tau * log(mean_t exp(x_t / tau)) per channel over chunk c's
 *                route tokens (route inputs default to q for r^q and k for r^k)
 *   gates        g_ij = sigmoid(<r^q_i, r^k_j> / sqrt(d) + bias), j < i (with window
 *                representatives: a log-sum-exp over chunk j's windows, see
 *                hla_config.pool_window), computed by
 *                a fixed binary32 recipe (a fused multiply-add wherever a product
 *                feeds a sum, exp/log evaluated by a fixed polynomial scheme) so
 *                that gates and skip decisions are reproducible bit for bit
 *   skip         j is skipped for query chunk i iff skip_threshold > 0 and
 *                g_ij < skip_threshold (equality is kept)
 *   composition  S <- 0; for active j ascending: S <- S + g_ij ((S A_j + B_j) - S)
 *   read-out     the token rule runs from that S over chunk i's tokens.
 *
 * Conventions
 *   - Every pointer argument named as device memory is a CUDA device pointer owned
 *     by the caller.  The library never allocates device memory: callers query
 *     the workspace and cache sizes and pass buffers in.
 *   - Every device pointer must be 16-byte aligned (HLA_ERR_INVALID_ARG otherwise),
 *     except the cache's n_chunks / m_partial counters (4-byte aligned).
 *   - Layouts are dense row-major:
 *       q, k, v, q_route, k_route, o : [B, T, H, d]      (dtype)
 *       alpha, beta                   : [B, T, H]         float32, alpha in (0,1], beta in [0,1]
 *                                       (alpha [B, T, H, d_k] with HLA_DECAY_CHANNEL)
 *       A_c                           : [d_k][d_k]; entry (r, c) multiplies column r
 *                                       of S into column c of S A
 *       B_c                           : [d_v][d_k]
 *   - q, k, v, the route inputs, o and cached A/B share the config's dtype.  Gates,
 *     pools and the composed state are float32.  Arithmetic is float32 (bf16
 *     tensor-core products accumulate in float32).
 *   - Calls are asynchronous on the given stream.  Argument checks run on the host
 *     before any launch; on error nothing is launched and hla_last_error() returns a
 *     message (thread-local).
 *   - Supported: C in {64, 128, 256}; d_k = d_v in {64, 128}; dtype float32 or
 *     bf16; any T >= 1 in prefill (a final partial chunk is read out and, with a
 *     cache, buffered).  The pages' default chunk is 256 tokens ("Main Findings",
 *     chunk-size ablation).  The WY solve and the intra-chunk read-out always work on
 *     64-token sub-chunks; at C > 64 the sub-chunk transitions are merged into the
 *     chunk's A_c, B_c (affine maps compose) and the composed state is carried to
 *     each sub-chunk, so pools, gates, skipping, composition and the decode cache are
 *     per chunk of C tokens.
 */
#ifndef HLA_H_
#define HLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same underlying type as cudaStream_t (NULL = legacy default stream). */
typedef struct CUstream_st* hla_stream_t;

typedef enum {
  HLA_OK = 0,
  HLA_ERR_INVALID_ARG = 1, /* NULL/misaligned pointer, inconsistent sizes      */
  HLA_ERR_UNSUPPORTED = 2, /* shape or dtype outside the supported set          */
  HLA_ERR_WORKSPACE = 3,   /* workspace or cache buffer too small              */
  HLA_ERR_CUDA = 4,        /* a CUDA runtime call failed (message has details) */
  HLA_ERR_TIMEOUT = 5      /* a bounded device-side wait expired (see below)   */
} hla_status;

typedef enum { HLA_F32 = 0, HLA_BF16 = 1 } hla_dtype;

typedef enum {
  HLA_GATES_ROUTED = 0, /* gates from the pools (the method)                        */
  HLA_GATES_ONE = 1,    /* every earlier chunk weight 1: native Gated DeltaNet      */
  HLA_GATES_ZERO = 2,   /* every earlier chunk weight 0: intra-chunk term only      */
  HLA_GATES_USER = 3    /* caller-given input-independent weights [B,H,N,N] (prefill) */
} hla_gate_mode;

/* Decay of the token rule.  SCALAR: S_t = S_{t-1} alpha_t (I - beta_t k_t k_t^T) +
 * beta_t v_t k_t^T (Gated DeltaNet).  CHANNEL: alpha_t is a vector over the d_k key
 * channels, S_t = S_{t-1} Diag(alpha_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T (the
 * KDA-style channel-wise decay named in the Gated DeltaNet-2 abstract on the HLA
 * listing page); with equal channels it is the scalar rule.  In CHANNEL mode the
 * chunk transitions and the intra-chunk read-out run the token rule row by row on
 * CUDA cores (rows of S evolve independently); the composition is unchanged. */
typedef enum { HLA_DECAY_SCALAR = 0, HLA_DECAY_CHANNEL = 1 } hla_decay_mode;

/* Storage of the closed chunks' transitions in a decode cache. */
typedef enum {
  HLA_CACHE_DENSE = 0,    /* A_j, B_j as d x d matrices (2 d^2 elements per chunk)        */
  HLA_CACHE_FACTORED = 1  /* the WY factors K_j, Wb_j, Ub_j (C x d each) and D_j, gamma_C:
                             A_j = gamma_C I - Wb_j^T D_j K_j, B_j = Ub_j^T D_j K_j
                             (3 C d elements; 25 % fewer bytes at C = 64, d = 128).
                             bf16 with d = 128 and C = 64 only (above C = 2d/3 the
                             factors are larger than A_j, B_j). */
} hla_cache_format;

typedef struct hla_config {
  int32_t B;              /* sequences                                          */
  int32_t H;              /* heads                                              */
  int32_t T;              /* tokens per sequence (prefill, transitions)         */
  int32_t C;              /* chunk size (64, 128 or 256)                        */
  int32_t dk, dv;         /* head dims, equal, 64 or 128                        */
  int32_t dtype;          /* hla_dtype                                          */
  int32_t gate_mode;      /* hla_gate_mode                                      */
  int32_t cache_format;   /* hla_cache_format of the caches used with this config */
  float tau;              /* pooling temperature, > 0                           */
  float bias;             /* gate bias b                                        */
  float skip_threshold;   /* <= 0: nothing skipped                              */
  int32_t pool_window;    /* 0: one key representative per chunk.  w > 0: the
                             pages' window representatives -- chunk j's key side is
                             W = C / w pools of w tokens each (w >= 8, w < C, w | C,
                             W <= 16) and the gate takes a log-sum-exp over them:
                             g_ij = sigmoid(log sum_u exp(<r^q_i, r^k_ju> / sqrt(d)) + b)
                             ("Methodology in Plain English" para. 2; "Main
                             Findings": window 32 by default)                   */
  int32_t decay_mode;     /* hla_decay_mode; CHANNEL takes alpha with a trailing
                             d_k axis and no factored cache                    */
} hla_config;

/*
 * Decode cache of B sequences (all pointers are device memory carved out of one
 * caller-owned block by hla_cache_init):
 *   A, Bm        [B, H, max_chunks, d, d]  dtype  -- transitions of closed chunks
 *                (HLA_CACHE_DENSE; NULL otherwise)
 *   Kf, Wf, Uf   [B, H, max_chunks, C, d]  dtype  -- K_j, Wb_j, Ub_j of closed chunks
 *   df           [B, H, max_chunks, C + 4] float32 -- gamma_C / gamma_t (t < C), then
 *                gamma_C, then padding (HLA_CACHE_FACTORED; all NULL otherwise)
 *   rk           [B, H, max_chunks, W, d]  float32 -- key pools of closed chunks (W = 1,
 *                or C / pool_window window pools)
 *   buf_k, buf_v, buf_qr, buf_kr  [B, H, C, d] dtype -- tokens of the open chunk
 *   buf_alpha, buf_beta           [B, H, C]  float32 (buf_alpha [B, H, C, d] if CHANNEL)
 *   n_chunks     [B] int32 -- closed chunks per sequence
 *   m_partial    [B] int32 -- tokens in the open chunk (0 .. C-1 between calls)
 * The cache is the resumable decode state ("Main Findings": per-chunk affine
 * states replace the KV cache): A/B take 2 d^2 elements per closed chunk.
 */
typedef struct hla_cache {
  int32_t max_chunks;
  int32_t B, H, C, d, dtype;
  int32_t format; /* hla_cache_format */
  int32_t pool_window; /* key representatives per closed chunk: 1, or C / pool_window */
  int32_t decay_mode;  /* hla_decay_mode (buf_alpha holds d_k values per token if CHANNEL) */
  void* A;
  void* Bm;
  void* Kf;
  void* Wf;
  void* Uf;
  float* df;
  float* rk;
  void* buf_k;
  void* buf_v;
  void* buf_qr;
  void* buf_kr;
  float* buf_alpha;
  float* buf_beta;
  int32_t* n_chunks;
  int32_t* m_partial;
} hla_cache;

/* Message for the last non-OK status returned on this thread ("" if none). */
const char* hla_last_error(void);

/* Bytes of the single device block that hla_cache_init carves (256-byte aligned
 * sub-buffers).  Returns 0 for an unsupported config. */
size_t hla_cache_bytes(const hla_config* cfg, int32_t max_chunks);

/* Fill *out with pointers into mem (device, >= hla_cache_bytes) and enqueue the
 * zeroing of the counters on stream.  Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE,
 * CUDA. */
hla_status hla_cache_init(const hla_config* cfg, int32_t max_chunks, void* mem, size_t bytes,
                          hla_cache* out, hla_stream_t stream);

/* View of sequences [b0, b0 + nb) of an initialised cache: *out gets B = nb and
 * every pointer advanced to sequence b0 (the buffers are sequence-major).  Host
 * only, nothing is launched.  Lets sequences of different prompt lengths be
 * prefilled one at a time into one cache, after which hla_decode_step advances
 * them together from their own positions.  Errors: INVALID_ARG. */
hla_status hla_cache_slice(const hla_cache* cache, int32_t b0, int32_t nb, hla_cache* out);

/* Workspace bytes that hla_prefill needs for cfg (0 for an unsupported config). */
size_t hla_prefill_workspace_bytes(const hla_config* cfg);

/* Workspace bytes that hla_decode_step needs for a cache of max_chunks chunks. */
size_t hla_decode_workspace_bytes(const hla_config* cfg, int32_t max_chunks);

/*
 * gdn_chunk_transitions -- the exact affine transition of every complete chunk
 * (Methodology para. 1), built through the chunkwise WY/UT form:
 *   l_t = sum_{s<=t} log alpha_s, gamma_t = exp(l_t), Gamma_ts = exp(l_t - l_s)
 *   L = strictly-lower(diag(beta) (Gamma o K K^T)), T = (I + L)^{-1} diag(beta)
 *   Wb = T diag(gamma) K, Ub = T V, D = diag(gamma_C / gamma_t)
 *   A_c = gamma_C I - Wb^T D K,  B_c = Ub^T D K.
 * In:  k, v [B,T,H,d] dtype; alpha, beta [B,T,H] float32 (device).
 * Out: A_out [B,H,T/C,d,d], B_out [B,H,T/C,d,d] dtype (device); a final partial
 *      chunk has no output.  Errors: INVALID_ARG, UNSUPPORTED, CUDA.
 * C = 64: the WY form above (tensor cores for bf16 with d = 128).  C > 64: this
 * call has no workspace for sub-chunk factors, so each chunk runs the token rule
 * row by row on CUDA cores (float32, exact in real arithmetic like the WY form);
 * hla_prefill builds the same transitions from 64-token WY sub-chunks instead.
 * HLA_DECAY_CHANNEL (alpha [B,T,H,d]): the token rule row by row at every C.
 */
hla_status gdn_chunk_transitions(const hla_config* cfg, const void* k, const void* v,
                                 const float* alpha, const float* beta, void* A_out,
                                 void* B_out, hla_stream_t stream);

/*
 * hla_routing -- pools and gates only (Overview; Methodology paras. 2 and 4).
 * In:  q_route, k_route [B,T,H,d] dtype (device; NULL is not allowed here).
 * Out: rq_out [B,H,N,d], rk_out [B,H,N*W,d] float32 (required), N = ceil(T/C), W = 1
 *      or C / pool_window (window u of chunk j at row j*W + u; windows past T unset);
 *      gates_out [B,H,N,N] float32 raw gates for j < i, 0 elsewhere (may be NULL);
 *      active_idx_out [B,H,N,N] int32: entries 0..cnt-1 of row i are the active j
 *      in ascending order, the rest are -1 (may be NULL together with cnt);
 *      active_cnt_out [B,H,N] int32.
 * Honours gate_mode (ONE/ZERO give 1/0 gates; USER is not accepted here).
 */
hla_status hla_routing(const hla_config* cfg, const void* q_route, const void* k_route,
                       float* rq_out, float* rk_out, float* gates_out,
                       int32_t* active_idx_out, int32_t* active_cnt_out, hla_stream_t stream);

/*
 * hla_gate_support -- routing diagnostics ("Key Contributions" 3; "Methodology in
 * Plain English" para. 4: a budget on the total routing mass and an order-2
 * effective number, the inverse sum of squares, of the chunks a query accesses).
 * For every query chunk i, over the chunks j < i kept by cfg->skip_threshold (all
 * of them for a threshold <= 0):
 *   mass_i = sum_j g_ij,   support_i = mass_i^2 / sum_j g_ij^2   (0 if none kept).
 * In:  gates [B,H,N,N] float32 (device), N = ceil(T/C): a gate matrix as written by
 *      hla_routing or hla_prefill (gates_out); only entries j < i are read.
 * Out: mass_out, support_out [B,H,N] float32 (device); either may be NULL, not both.
 * float32 sums (per-lane partial sums combined by a butterfly).
 * Errors: INVALID_ARG, UNSUPPORTED, CUDA.
 */
hla_status hla_gate_support(const hla_config* cfg, const float* gates, float* mass_out, float* support_out,
                            hla_stream_t stream);

/*
 * hla_prefill -- HLA over a whole prompt (Key Contributions 3; Methodology paras. 1-4).
 * In:  q, k, v [B,T,H,d] dtype; alpha, beta [B,T,H] float32;
 *      q_route, k_route [B,T,H,d] dtype or NULL (NULL: q, k);
 *      user_gates [B,H,N,N] float32 (HLA_GATES_USER only, else ignored).
 * Out: o [B,T,H,d] dtype.  Optional (NULL to skip): gates_out, active_idx_out,
 *      active_cnt_out as in hla_routing; cache_out -- an initialised cache with
 *      max_chunks >= T/C, filled with A/B/rk of every complete chunk, the final
 *      partial chunk's tokens and the counters.
 * workspace: device, >= hla_prefill_workspace_bytes(cfg), 256-byte aligned.
 * Path: routing on a library side stream (forked from and joined back to `stream`
 * by events) beside the chunk transitions; then the composition and the read-out.
 * The side stream is one per device, made on the first call (and again when a
 * different CUDA context is current), and one process-wide lock is held while a
 * call enqueues its fork, routing and join: concurrent calls on different streams
 * are correct, but their routing stages run one after another on that stream.
 * Every return after the fork, an error included, leaves `stream` joined to it.
 * With HLA_DECAY_CHANNEL and bf16, d = 128, the transitions and the read-out run on
 * the tensor cores with the decays folded into prepared keys and queries per 64-token
 * sub-chunk (k o gamma_t, k / gamma_t, k o gamma_C / gamma_t, q o gamma_t with
 * gamma_t the decay accumulated since the sub-chunk's first token, per channel).
 * Their range: in every channel the decay over one sub-chunk must stay above e^-80
 * (k / gamma_t stays finite); a prefill that leaves it records code 0x8, reported by
 * hla_device_status.  With float32 or d = 64 they run the token rule per chunk on CUDA
 * cores (no such limit).
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA.
 */
hla_status hla_prefill(const hla_config* cfg, const void* q, const void* k, const void* v,
                       const float* alpha, const float* beta, const void* q_route,
                       const void* k_route, const float* user_gates, void* o,
                       float* gates_out, int32_t* active_idx_out, int32_t* active_cnt_out,
                       hla_cache* cache_out, void* workspace, size_t workspace_bytes,
                       hla_stream_t stream);

/*
 * hla_decode_step -- one new token per sequence (Key Contributions 3: dynamic
 * autoregressive decoding; Methodology para. 4: skipped chunks are not read).
 * In:  q, k, v [B,H,d] dtype; alpha, beta [B,H] float32 (alpha [B,H,d] with channel-wise
 *      decay); q_route, k_route [B,H,d]
 *      or NULL (q, k).  cache: initialised (by hla_prefill or empty).
 * Out: o [B,H,d] dtype.  The token is appended to the open chunk; the query pool
 *      runs over the open chunk's m tokens so far; gates against every closed
 *      chunk's key pool; active chunks are applied by the equivalent right-to-left
 *      form  y += g_j B_j x; x <- (1-g_j) x + g_j A_j x  (j descending), which reads
 *      each active A_j/B_j once; when the open chunk reaches C tokens it is closed
 *      (its A/B/rk are appended; at C = 64 by the WY form, at C > 64 by the token
 *      rule run row by row).  Gate modes ROUTED, ONE and ZERO.
 * workspace: device, >= hla_decode_workspace_bytes(cfg, cache->max_chunks): the
 *      active lists and gates ([B,H,max_chunks] int32 and float32) and one list length
 *      per (sequence, head), each part rounded up to 256 bytes.
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE (also: cache full), CUDA.
 */
hla_status hla_decode_step(const hla_config* cfg, hla_cache* cache, const void* q,
                           const void* k, const void* v, const float* alpha,
                           const float* beta, const void* q_route, const void* k_route,
                           void* o, void* workspace, size_t workspace_bytes,
                           hla_stream_t stream);

/*
 * hla_decode_step_static -- hla_decode_step without a caller workspace.
 * The pages have no counterpart to this call: it exists for callers that may not
 * allocate device memory where they decode (a plug-in inside a runtime that owns
 * all device memory through its own pool, or a thread with no allocator in
 * reach).  Same arguments, layouts, semantics and errors as hla_decode_step, minus
 * the workspace: the scratch is a fixed device array inside this library,
 * HLA_DECODE_STATIC_SCRATCH_BYTES long: it holds hla_decode_workspace_bytes(cfg,
 * max_chunks) when 8 B per (sequence, head, chunk) plus 4 B per (sequence, head), each
 * part rounded up to 256 B, fit in it (for example B*H = 1024 with max_chunks = 1023).
 * A larger cache is rejected with HLA_ERR_WORKSPACE before anything is launched.
 * No call allocates or frees device memory.
 * Set-up: the first call on a device (the current one) looks up the array's
 * device address and keeps it; make that first call before any stream capture.
 * The address belongs to the CUDA context current at that call.  A call under a
 * different context (a non-primary context, or the primary context recreated by
 * cudaDeviceReset) looks it up again, which is again a set-up call: make it
 * outside stream capture too.
 * Sharing: every call on a device writes the same array.  Nothing in it has to
 * start at zero, but calls whose kernels may overlap in time (different streams
 * or host threads) race on it; serialise them.
 */
#define HLA_DECODE_STATIC_SCRATCH_BYTES ((size_t)8 << 20)
hla_status hla_decode_step_static(const hla_config* cfg, hla_cache* cache, const void* q,
                                  const void* k, const void* v, const float* alpha,
                                  const float* beta, const void* q_route,
                                  const void* k_route, void* o, hla_stream_t stream);

/*
 * Bounded device waits.  Kernels that wait on an mbarrier or a flag give up after
 * a fixed number of polls, record a code in a device-side error word and return.
 * hla_device_status synchronises the device, reads and (if clear != 0) resets that
 * word; it returns HLA_ERR_TIMEOUT if a wait expired since the last reset (code bit
 * 0x1, or 0x2 for a tensor-memory allocation), HLA_ERR_WORKSPACE if a decode step
 * found its cache full (0x4), HLA_ERR_UNSUPPORTED if a prefill with a decay per
 * channel left the tensor-core range described at hla_prefill (0x8), else HLA_OK (or
 * HLA_ERR_CUDA).  *code_out (may be NULL) receives the raw word.
 */
hla_status hla_device_status(int32_t clear, uint32_t* code_out);

/*
 * Bounded-wait check (diagnostic).  Enqueues on stream one kernel that waits on an
 * mbarrier with the library's bounded wait.  complete != 0: the barrier is
 * completed before the wait, which returns at once.  complete == 0: nothing
 * completes it, so the wait gives up after limit_us microseconds, records the
 * timeout in the device error word and the kernel exits normally; the next
 * hla_device_status returns HLA_ERR_TIMEOUT (code bit 0x1) and the context stays
 * usable.  limit_us in [1, 100000].  Errors: INVALID_ARG, CUDA.
 */
hla_status hla_check_bounded_wait(uint32_t limit_us, int32_t complete, hla_stream_t stream);

/*
 * Stage timing (tracing).  While enabled, hla_prefill and hla_decode_step record a
 * pair of CUDA events on the caller's stream around each stage below and count the
 * kernels each stage launches.  hla_profile_read synchronises the device, writes
 * the accumulated milliseconds and launch counts per stage into ms_out[] and
 * launches_out[] (HLA_STAGE_COUNT entries each; either may be NULL) and, if
 * reset != 0, clears them.  Errors: CUDA.
 */
typedef enum {
  HLA_STAGE_POOLS = 0,        /* log-mean-exp pools                        */
  HLA_STAGE_GATES = 1,        /* gates + active lists                      */
  HLA_STAGE_TRANSITIONS = 2,  /* chunk transitions (A, B) and WY factors   */
  HLA_STAGE_COMPOSE = 3,      /* gated composition of S_in                 */
  HLA_STAGE_READOUT = 4,      /* intra-chunk read-out                      */
  HLA_STAGE_CACHE = 5,        /* prefill -> decode cache hand-off          */
  HLA_STAGE_DECODE = 6,       /* decode: sweep, gates, active chain        */
  HLA_STAGE_DECODE_CLOSE = 7, /* decode: closing full chunks, counters     */
  HLA_STAGE_CHAIN = 8,        /* C > 64: sub-chunk transitions merged per
                                 chunk, states advanced to sub-chunks      */
  HLA_STAGE_COUNT = 9
} hla_stage;

hla_status hla_profile_enable(int32_t on);
hla_status hla_profile_read(float* ms_out, int32_t* launches_out, int32_t reset);

#ifdef __cplusplus
}
#endif
#endif /* HLA_H_ */
