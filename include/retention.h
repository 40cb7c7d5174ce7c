/*
 * retention.h — C ABI of libretention.so, the Multi-Scale Retention (MSR) hot
 * path for NVIDIA B200 (sm_100a).
 *
 * What is computed.  For one head with fixed decay gamma in [0, 1], queries
 * q_n, keys k_n (rows of length d_k) and values v_n (rows of length d_v):
 *
 *     o_n = sum_{m <= n} gamma^(n-m) (q_n . k_m) v_m                      (R)
 *
 * Sources, by page title and section:
 *   - abeam.tech summary of Sun et al. 2023, "Retentive Network: A Successor to
 *     Transformer for Large Language Models":
 *       「Retentionは「内容に応じた参照」と「距離による忘却」を掛け合わせる」 — (R):
 *         values of past positions weighted by Q_n K_m^T and gamma^(n-m),
 *         future masked;
 *       「学習は並列、生成は状態更新」 — the parallel form (Q K^T * D) V with the
 *         causal decay mask D_nm = gamma^(n-m) [n >= m], and the recurrent
 *         form S_n = gamma S_(n-1) + K_n^T V_n, o_n = Q_n S_n;
 *       「長文の学習にはチャンク再帰を使う」 — the chunkwise form: parallel inside
 *         a chunk, past chunks through the state updated at each chunk end;
 *       「多時間尺度・ゲート・正規化で表現力を補う」 — one fixed gamma per head,
 *         a Swish gate and a per-head GroupNorm.
 *   - mlnews.online abstract page for arXiv 2307.08621, summary bullets —
 *     GroupNorm per head before the heads are concatenated.
 *   - eulerwa.com tutorial "3. RetNet 상세", section "장점" — the three forms
 *     give the same values.
 *
 * No 1/sqrt(d_k) factor is applied inside retention (the pages' formula has
 * none); callers fold any scale into q or k.  Rotary position encoding, if
 * used, is applied to q and k before these calls (retention_rope).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *   Memory:   every tensor argument is a DEVICE pointer on the current CUDA
 *             device, owned by the caller, 16-byte aligned, densely packed in
 *             the row-major layout stated below.  The library never frees or
 *             keeps a caller pointer after the call returns.  `gamma` is the one
 *             HOST array: it is read during the call and not retained.
 *   Layout:   token-major.  q, k: [B, T, H, d_k]; v: [B, T, H, d_v];
 *             outputs o / y: [B, T, H, d_v]; gate g: [B, T, H * d_v];
 *             states: [B (or nseq, or N), H, d_k, d_v] float32, row = d_k index.
 *   Dtypes:   RET_F32 (float) or RET_BF16 (bfloat16, stored as uint16).
 *             bf16 inputs are multiplied on tensor cores with float32
 *             accumulation; the carried state is always float32.
 *   Gamma:    host double[H], each 0 <= gamma_h <= 1 (0^0 = 1: gamma = 0
 *             keeps only the diagonal term q_n.k_n v_n).  H <= 64.
 *   Streams:  every call only enqueues work on `stream` (a cudaStream_t; NULL
 *             = the legacy default stream) and returns without synchronising.
 *             The returned status covers argument validation and launch
 *             errors; faults and time-outs detected on the device are
 *             reported later by retention_check_device_error().
 *   Errors:   a validation status (RET_ERR_INVALID_ARG, RET_ERR_UNSUPPORTED,
 *             RET_ERR_WORKSPACE) means nothing was enqueued and no output was
 *             touched; RET_ERR_CUDA means a launch failed and earlier kernels
 *             of the same call may have run.  RET_ERR_UNSUPPORTED means the
 *             arguments are valid but the library has no kernel for the
 *             shape or dtype combination; there is no fallback path.
 *   Aliasing: outputs must not overlap inputs, except that
 *             retention_recurrent_step(s) update `state` in place by design
 *             and retention_rope may rotate q and k in place.
 */
#ifndef RETENTION_H_
#define RETENTION_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define RETENTION_ABI_VERSION 3

#if defined(__GNUC__)
#define RET_API __attribute__((visibility("default")))
#else
#define RET_API
#endif

typedef struct CUstream_st* ret_stream_t; /* == cudaStream_t */

typedef enum {
  RET_OK = 0,
  RET_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size, gamma out of [0,1] */
  RET_ERR_UNSUPPORTED = 2,   /* valid request with no kernel in the library */
  RET_ERR_CUDA = 3,          /* a CUDA runtime/driver call failed */
  RET_ERR_TIMEOUT = 4,       /* a bounded device-side wait expired (from check_device_error) */
  RET_ERR_WORKSPACE = 5,     /* workspace missing or smaller than the size query returned */
  RET_ERR_DEVICE_DATA = 6,   /* device-resident metadata (cu_seqlens) was inconsistent */
  RET_ERR_RANGE = 7          /* a tensor-core operand exceeded fp16's range (from check_device_error) */
} ret_status;

typedef enum { RET_F32 = 0, RET_BF16 = 1 } ret_dtype;

/*
 * Per-head GroupNorm followed by the Swish gate (abeam.tech summary,
 * 「多時間尺度・ゲート・正規化で表現力を補う」; mlnews.online abstract page,
 * summary bullets).  For each token t and head h, over the d_v channels c:
 *     mu = mean_c o[t,h,c];  var = mean_c (o[t,h,c] - mu)^2   (biased)
 *     y[t,h,c] = ((o - mu) / sqrt(var + eps) * weight[h*d_v+c] + bias[h*d_v+c])
 *                * g[t, h*d_v+c] * sigmoid(g[t, h*d_v+c])
 */
typedef struct {
  const void*  g;        /* device gate [ntok, H*d_v], dtype g_dtype (required) */
  ret_dtype    g_dtype;
  const float* weight;   /* device [H*d_v] float32, or NULL for 1 */
  const float* bias;     /* device [H*d_v] float32, or NULL for 0 */
  float        eps;      /* added to the variance; must be >= 0 and finite */
} ret_norm_gate;

/* ABI version of the loaded library (RETENTION_ABI_VERSION at build time). */
RET_API int retention_abi_version(void);

/* SHA-256, as 64 hex digits, of the sources the library was built from (the
 * kernel sources and this header), or "unknown" for a build that did not pass
 * it.  Static string, owned by the library.  The Python binding compares it
 * with the source tree next to it and refuses a library built from other
 * sources. */
RET_API const char* retention_source_sha(void);

/* Static, human-readable name of a status code. */
RET_API const char* retention_status_string(ret_status status);

/*
 * Parallel form O = (Q K^T * D) V, D_nm = gamma_h^(n-m) for n >= m else 0
 * (abeam.tech summary, 「学習は並列、生成は状態更新」).  Every (b, h) pair is an
 * independent causal sequence of T tokens.
 *   q, k:  [B,T,H,dk] in_dtype      v: [B,T,H,dv] in_dtype
 *   o:     [B,T,H,dv] o_dtype (fully overwritten)
 *   workspace: device scratch of at least retention_parallel_workspace_size()
 *          bytes, 256-byte aligned, owned by the caller; NULL when that size
 *          is 0.  Its contents on entry do not matter.
 * Kernels:
 *   - bf16 inputs with dk in {64,128,256} and dv in {64,128,256,512}: tensor
 *     cores.  An fp16 copy of v goes to the workspace (exact for |v| < 2^16;
 *     larger values are reported as RET_ERR_RANGE by
 *     retention_check_device_error), then 128-row query tiles run against
 *     every causal 128-key block with the scores and decay formed in f32,
 *     rounded once to fp16 for the P V product, f32 accumulation.  Precision
 *     and range as the chunkwise tensor-core path.  The workspace also holds
 *     a tile counter (its last 256 bytes): tiles cost 1 to T/128 key blocks,
 *     so the persistent kernel hands them out in a dynamic order.  Calls
 *     that share one workspace must be ordered (one stream).
 *   - otherwise (float32 inputs, or bf16 with other head dims): CUDA cores,
 *     float32 arithmetic, dk and dv up to 256.
 * Supported: T >= 1; B*T*H*max(dk,dv) < 2^31.
 * Returns RET_ERR_INVALID_ARG for null pointers, B,T,H,dk,dv < 1, H > 64 or
 * gamma outside [0,1]; RET_ERR_UNSUPPORTED for head dims no kernel takes;
 * RET_ERR_WORKSPACE when the workspace is needed and missing, too small or
 * not 256-byte aligned.
 */
RET_API size_t retention_parallel_workspace_size(ret_dtype in_dtype, int B, int T, int H,
                                                 int dk, int dv);
RET_API ret_status retention_parallel_fwd(const void* q, const void* k, const void* v,
                                  ret_dtype in_dtype, const double* gamma,
                                  void* o, ret_dtype o_dtype,
                                  void* workspace, size_t workspace_bytes,
                                  int B, int T, int H, int dk, int dv,
                                  ret_stream_t stream);

/*
 * Bytes of device workspace retention_chunkwise_fwd needs for these sizes
 * (0 if the arguments are invalid).  The workspace holds the state entering
 * every chunk (float32 for float32 inputs; fp16 for bf16 inputs, which also
 * keep an fp16 copy of v there, T*H*dv values); its contents need no
 * initialisation and are scratch after the call.  `nseq` = 0 for the padded
 * layout, else the number of packed sequences (then B must be 1 and T is the
 * total token count).
 */
RET_API size_t retention_chunkwise_workspace_size(ret_dtype in_dtype, int chunk,
                                          int B, int T, int H, int dk, int dv,
                                          int nseq);

/*
 * The chunk length the chunkwise kernels evaluate for a requested `chunk`
 * (every chunk length gives the same result, see retention_chunkwise_fwd):
 * `chunk` itself for float32 inputs; for bf16 inputs 128 tokens, or 256 when
 * dv >= 256, whatever chunk was requested (the length the tensor-core kernels
 * run fastest at).  Returns 0 for unsupported arguments.  No counterpart on
 * the pages: it lets a caller count the work the kernels do.
 */
RET_API int retention_chunkwise_executed_chunk(ret_dtype in_dtype, int chunk, int dk, int dv);

/*
 * Chunkwise recurrent form (abeam.tech summary, 「長文の学習にはチャンク再帰を
 * 使う」), with an optional fused GroupNorm + Swish-gate epilogue.  For a
 * chunk of L <= `chunk` tokens starting at token s (row i = n - s):
 *     O[i] = sum_{j<=i} gamma^(i-j) (q_i . k_j) v_j + gamma^(i+1) q_i S_prev
 *     S    = gamma^L S_prev + sum_j gamma^(L-1-j) k_j^T v_j
 * which equals (R) exactly in real arithmetic for every chunk length.
 *
 *   q, k:  [B,T,H,dk] in_dtype      v: [B,T,H,dv] in_dtype
 *   cu_seqlens: NULL for B independent sequences of T tokens each; otherwise
 *          a DEVICE int32 [nseq+1] of packed sequence offsets (B must be 1,
 *          cu_seqlens[0] = 0, non-decreasing, cu_seqlens[nseq] = T).  Each
 *          sequence starts from its own state and its chunks start at its
 *          first token; empty sequences are allowed.  If the device array
 *          breaks these rules the kernels clamp every access to [0, T) and
 *          raise RET_ERR_DEVICE_DATA through retention_check_device_error().
 *   state_in:  [nseq or B, H, dk, dv] float32, or NULL for zeros.
 *   state_out: [nseq or B, H, dk, dv] float32 final states, or NULL.  An empty
 *          sequence's state_out equals its state_in (or zeros).
 *   out:   [B,T,H,dv] o_dtype.  With ng == NULL it receives the retention
 *          output o; with ng != NULL it receives y = GroupNorm(o) * swish(g).
 *   workspace: device scratch of at least
 *          retention_chunkwise_workspace_size(...) bytes, 256-byte aligned.
 * Supported:
 *   in_dtype RET_F32: dk, dv in 1..256, any chunk >= 1 (CUDA-core float32).
 *   in_dtype RET_BF16: tensor-core kernels (tcgen05, TMEM accumulators), dk in
 *          {64, 128, 256}, dv in {64, 128, 256, 512}, chunk in
 *          {64, 128, 256, 512}; other bf16 shapes return
 *          RET_ERR_UNSUPPORTED.  Every requested chunk is evaluated as
 *          chunks of 128 tokens (256 when dv >= 256), which yields the same
 *          result up to rounding (retention_chunkwise_executed_chunk).
 *   out dtype RET_F32 or RET_BF16; H <= 64; T*H*max(dk,dv) < 2^31.
 * Precision of the bf16 path: q and k enter the MMAs as they are, v as its
 *   fp16 value (exact inside fp16's range); the decayed scores, the decayed
 *   query rows gamma^(i+1) q_i, zeta*K and the carried state are rounded to
 *   fp16 (11 significant bits) before their MMAs; every product accumulates
 *   in float32 and the state is carried in float32 between chunks.  A value
 *   outside fp16's range (|v| >= 2^16, a decayed score or state entry beyond
 *   65504) is reported as RET_ERR_RANGE by retention_check_device_error().
 */
RET_API ret_status retention_chunkwise_fwd(const void* q, const void* k, const void* v,
                                   ret_dtype in_dtype, const double* gamma,
                                   int chunk,
                                   const int32_t* cu_seqlens, int nseq,
                                   const float* state_in, float* state_out,
                                   void* out, ret_dtype out_dtype,
                                   const ret_norm_gate* ng,
                                   void* workspace, size_t workspace_bytes,
                                   int B, int T, int H, int dk, int dv,
                                   ret_stream_t stream);

/*
 * The two phases of retention_chunkwise_fwd as separate calls (same argument
 * meanings and rules).  retention_chunkwise_states runs the chunk-to-chunk
 * recurrence of the state (abeam.tech summary, 「長文の学習にはチャンク再帰を使う」:
 * the state is updated at the end of every chunk): it stores the state
 * entering every chunk in `workspace` and writes the final states to
 * `state_out` (optional).  Alone, it is a prefill that yields the decode
 * state without computing outputs.  retention_chunkwise_outputs then reads
 * that workspace and writes `out` (o, or y when `ng` is given); it must
 * follow a states call with identical q/k/v-independent arguments (dtype,
 * gamma, chunk, cu_seqlens, sizes) on the same stream, with the workspace
 * untouched in between.  `has_state_in` is nonzero when that states call was
 * given a state_in.  Together they do exactly what retention_chunkwise_fwd
 * does.
 */
RET_API ret_status retention_chunkwise_states(const void* k, const void* v, ret_dtype in_dtype,
                                              const double* gamma, int chunk,
                                              const int32_t* cu_seqlens, int nseq,
                                              const float* state_in, float* state_out,
                                              void* workspace, size_t workspace_bytes,
                                              int B, int T, int H, int dk, int dv,
                                              ret_stream_t stream);

RET_API ret_status retention_chunkwise_outputs(const void* q, const void* k, const void* v,
                                               ret_dtype in_dtype, const double* gamma,
                                               int chunk, const int32_t* cu_seqlens, int nseq,
                                               int has_state_in, void* out, ret_dtype out_dtype,
                                               const ret_norm_gate* ng, const void* workspace,
                                               size_t workspace_bytes, int B, int T, int H,
                                               int dk, int dv, ret_stream_t stream);

/*
 * retention_chunkwise_fwd for callers that cannot allocate device memory.
 * The paper has no counterpart: this is a deployment convenience.  Some
 * callers have no allocator to hand: code that runs where cudaMalloc is not
 * allowed or would stall (inside a memory pool's own bookkeeping, in embedded
 * runtimes with a fixed device budget, or wherever the process must not grow
 * its device footprint after start-up).  This entry point takes the same
 * arguments as retention_chunkwise_fwd except the workspace: it uses a
 * scratch array compiled into the library instead, and it allocates nothing
 * (no cudaMalloc, no cudaFree, no allocating library call).
 *   - The scratch array holds RETENTION_STATIC_WORKSPACE_BYTES on every GPU
 *     that loads this library, for as long as the library stays loaded.
 *   - A request whose retention_chunkwise_workspace_size() exceeds that
 *     capacity returns RET_ERR_WORKSPACE and enqueues nothing; other
 *     validation errors are those of retention_chunkwise_fwd.
 *   - The first call on a device looks up the array's device address (one
 *     cudaGetSymbolAddress per device, cached); make that first call before
 *     any stream capture.
 *   - Every call on a device shares the one array and leaves its contents
 *     behind; nothing in it needs to start at zero.  Calls that overlap on the
 *     GPU (different streams, or several host threads) race on the array and
 *     must be serialised by the caller.
 * Outputs equal those of retention_chunkwise_fwd on the same arguments.
 */
#define RETENTION_STATIC_WORKSPACE_BYTES ((size_t)32 << 20)

RET_API ret_status retention_chunkwise_fwd_static_ws(const void* q, const void* k,
                                                     const void* v, ret_dtype in_dtype,
                                                     const double* gamma, int chunk,
                                                     const int32_t* cu_seqlens, int nseq,
                                                     const float* state_in, float* state_out,
                                                     void* out, ret_dtype out_dtype,
                                                     const ret_norm_gate* ng,
                                                     int B, int T, int H, int dk, int dv,
                                                     ret_stream_t stream);

/*
 * One recurrent decode step for N independent sequences (abeam.tech summary,
 * 「学習は並列、生成は状態更新」): for every (n, h), in this order,
 *     S <- gamma_h S + k^T v      (state updated in place)
 *     o  = q S                     (read after the update)
 *   q, k: [N,H,dk] in_dtype   v: [N,H,dv] in_dtype
 *   state: [N,H,dk,dv] float32, read and overwritten
 *   o: [N,H,dv] o_dtype
 * Supported: dk in 1..1024, dv in 1..4096; the state streams through HBM once
 * (read + write), the memory-bound part of generation.
 */
RET_API ret_status retention_recurrent_step(const void* q, const void* k, const void* v,
                                    ret_dtype in_dtype, const double* gamma,
                                    float* state, void* o, ret_dtype o_dtype,
                                    int N, int H, int dk, int dv,
                                    ret_stream_t stream);

/*
 * Tn consecutive recurrent decode steps for N independent sequences in one
 * pass over the state (the recurrence of retention_recurrent_step applied Tn
 * times; abeam.tech summary, 「学習は並列、生成は状態更新」, with the sum
 * unrolled as in the chunkwise form of 「長文の学習にはチャンク再帰を使う」):
 *     o_t = gamma^(t+1) q_t S + sum_{j<=t} gamma^(t-j) (q_t . k_j) v_j
 *     S  <- gamma^Tn S + sum_j gamma^(Tn-1-j) k_j^T v_j
 * for t = 0..Tn-1, with S the state entering the call.  The state is read and
 * written once for all Tn tokens (speculative or prompt-continuation steps).
 *   q, k: [N,Tn,H,dk] in_dtype   v: [N,Tn,H,dv] in_dtype   (token-major)
 *   state: [N,H,dk,dv] float32, read and overwritten
 *   o: [N,Tn,H,dv] o_dtype
 * Supported: 1 <= Tn <= 16, dk and dv multiples of 4 with dk <= 512 and
 * dv <= 4096; otherwise RET_ERR_UNSUPPORTED.  Two paths, chosen per call:
 *   tensor cores: in_dtype RET_BF16, Tn >= 12, dk in {128, 256}, dv a
 *     multiple of 128 whose operand tiles fit in shared memory (up to 512 at
 *     dk = 256, 768 at dk = 128).  The two products that touch every state
 *     element run as tcgen05 MMAs of kind::tf32 on the float32 state (operands
 *     read at tf32 precision, relative 2^-11; the state itself stays float32):
 *     results are within the bf16-input tolerance.  Needs a device error word
 *     (retention_check_device_error reports a bounded wait that ran out).
 *   CUDA cores: every other case, float32 FMAs (exact to float32 rounding).
 * Both are bound by the state's HBM traffic.
 */
RET_API ret_status retention_recurrent_steps(const void* q, const void* k, const void* v,
                                             ret_dtype in_dtype, const double* gamma,
                                             float* state, void* o, ret_dtype o_dtype,
                                             int N, int Tn, int H, int dk, int dv,
                                             ret_stream_t stream);

/*
 * Backward of the chunkwise form: the gradients for training in the parallel
 * form (eulerwa.com tutorial "3. RetNet 상세", section "장점"; the pages state
 * the forward only, these are its derivatives).  For each sequence and head,
 * with the forward started from S0 = state_in (zero if NULL),
 *     o_n = sum_{m<=n} gamma^(n-m) (q_n . k_m) v_m + gamma^(n+1) q_n S0
 *     S_T = gamma^T S0 + sum_m gamma^(T-1-m) k_m^T v_m
 * and upstream gradients dO = d_out and dS_T = d_state_out (zero if NULL):
 *     dq_n = sum_{m<=n} gamma^(n-m) (dO_n . v_m) k_m + gamma^(n+1) dO_n S0^T
 *     dk_m = sum_{n>=m} gamma^(n-m) (dO_n . v_m) q_n + gamma^(T-1-m) v_m dS_T^T
 *     dv_m = sum_{n>=m} gamma^(n-m) (q_n . k_m) dO_n + gamma^(T-1-m) k_m dS_T
 *     dS0  = sum_n gamma^(n+1) q_n^T dO_n + gamma^T dS_T      (-> d_state_in)
 * evaluated chunk by chunk (`chunk` tokens; any length gives the same values):
 * a forward pass over the chunks carries S, a backward pass carries the state
 * of everything after each chunk.  This is the gradient of the raw retention
 * output o; the GroupNorm and gate, when used, are differentiated by the caller.
 *   q, k: [B,T,H,dk] in_dtype   v, d_out: [B,T,H,dv] in_dtype (same layout and
 *   packing as retention_chunkwise_fwd, incl. cu_seqlens/nseq)
 *   state_in, d_state_out: [nseq|B,H,dk,dv] float32 or NULL
 *   dq, dk: [B,T,H,dk] float32   dv: [B,T,H,dv] float32   (written in full)
 *   d_state_in: [nseq|B,H,dk,dv] float32 or NULL (not emitted)
 *   workspace: caller-owned device buffer, 256-byte aligned, at least
 *     retention_chunkwise_bwd_workspace_size(...) bytes (chunk offsets and two
 *     float32 states per chunk); RET_ERR_WORKSPACE otherwise.
 * Supported: in_dtype RET_F32 or RET_BF16, dk and dv in 1..256, any chunk >= 1;
 * and bf16 with dk in {64, 128, 256}, dv = 512 on the tensor cores.
 * Two paths, chosen per call:
 *   tensor cores: in_dtype RET_BF16 with dk in {64, 128, 256}, dv in {64, 128,
 *     256, 512} and a chunk of 64..512.  The three gradients are three
 *     retentions with the operand roles exchanged, on the forward's tcgen05
 *     kernels with the forward's precision (fp16 operands, float32
 *     accumulation): dQ causal from S0^T; dV and dK anti-causal (the chunks
 *     walked last to first, each carrying the state of everything after it),
 *     started from dS_T and dS_T^T, the dV pass's final state being dS0.
 *     With dv = 512 the dQ and dK retentions, whose scores contract over dv,
 *     each run as two passes over the halves of dv, the second adding to the
 *     first.  `chunk` only selects the layout, the kernels' own chunk is used.
 *   CUDA cores: every other supported case; every product and sum is float32
 *     (bf16 inputs are widened exactly).
 * Other heads return RET_ERR_UNSUPPORTED.  The workspace size query returns 0
 * for arguments the call would reject, and otherwise the larger of the two
 * paths' needs.
 */
RET_API size_t retention_chunkwise_bwd_workspace_size(ret_dtype in_dtype, int chunk, int B,
                                                      int T, int H, int dk, int dv, int nseq);
RET_API ret_status retention_chunkwise_bwd(const void* q, const void* k, const void* v,
                                           const void* d_out, ret_dtype in_dtype,
                                           const double* gamma, int chunk,
                                           const int32_t* cu_seqlens, int nseq,
                                           const float* state_in, const float* d_state_out,
                                           float* dq, float* dk, float* dv, float* d_state_in,
                                           void* workspace, size_t workspace_bytes,
                                           int B, int T, int H, int dk_, int dv_,
                                           ret_stream_t stream);

/*
 * Rotary position encoding of q and k, applied before the retention calls.
 * The abeam.tech summary (section 「Retentionは「内容に応じた参照」と「距離による
 * 忘却」を掛け合わせる」) rotates Q and K by position after the projections and
 * eulerwa.com "3. RetNet 상세" ("장점") calls retention RoPE-compatible; the
 * pages give no formula, and this is the standard rotary form: for a token at
 * position p (its index within its own sequence) and pair i < d/2,
 *     x'[2i]   = x[2i] cos(p theta_i) - x[2i+1] sin(p theta_i)
 *     x'[2i+1] = x[2i] sin(p theta_i) + x[2i+1] cos(p theta_i),
 *     theta_i  = base^(-2i/d)                                   (base > 1)
 *   q, k: [B,T,H,d] dtype (packed: B = 1 with cu_seqlens/nseq as for
 *   retention_chunkwise_fwd; positions restart at every sequence)
 *   q_out, k_out: [B,T,H,d] dtype, written in full; q_out may equal q and
 *   k_out may equal k (in place), no other overlap.
 * The angle is reduced modulo 2 pi in double precision, the rotation is
 * float32 and a bf16 output is rounded to nearest once.  d even, any H.
 */
RET_API ret_status retention_rope(const void* q, const void* k, ret_dtype dtype, void* q_out,
                                  void* k_out, double base, const int32_t* cu_seqlens, int nseq,
                                  int B, int T, int H, int d, ret_stream_t stream);

/*
 * Residual linear attention (RLA), the variant on the RAttention page (section
 * "Residual Linear Attention (RLA) 수식"): per sequence and head, a state
 * without decay read w = `window` tokens late,
 *     S_t = S_(t-1) + phi(k_t)^T v_t,      o_t = phi(q_t) S_(t-w-1)
 * (S of a position before the sequence is zero, so o_t = 0 for the first w+1
 * tokens).  phi is the softmax over the head dimension (the page names a
 * softmax-based feature map the best choice and gives no formula).  This is
 * the retention (R) at gamma = 1 on phi(q), phi(k_(t-w-1)), v_(t-w-1), and it
 * runs on the same kernels: one pass maps and shifts the inputs into the
 * workspace (stored in in_dtype), then the chunkwise forward.  The local
 * sliding-window attention the page pairs it with is not part of this call.
 *   q, k: [B,T,H,dk] in_dtype   v: [B,T,H,dv] in_dtype (packed sequences as
 *   for retention_chunkwise_fwd)     o: [B,T,H,dv] o_dtype, written in full
 *   window >= 0; workspace: >= retention_rla_workspace_size(...) bytes,
 *   256-byte aligned (RET_ERR_WORKSPACE otherwise).
 * Supported: the shapes of retention_chunkwise_fwd (bf16 on tensor cores, f32
 * on CUDA cores).
 */
RET_API size_t retention_rla_workspace_size(ret_dtype in_dtype, int B, int T, int H, int dk,
                                            int dv, int nseq);
RET_API ret_status retention_rla_fwd(const void* q, const void* k, const void* v,
                                     ret_dtype in_dtype, int window, const int32_t* cu_seqlens,
                                     int nseq, void* o, ret_dtype o_dtype, void* workspace,
                                     size_t workspace_bytes, int B, int T, int H, int dk, int dv,
                                     ret_stream_t stream);

/*
 * Chunkwise forward with the rotary position encoding of q and k in the same
 * call: the result of retention_rope(q, k, base) followed by
 * retention_chunkwise_fwd on the rotated q and k, bit for bit (abeam.tech
 * summary, 「Retentionは「内容に応じた参照」と「距離による忘却」を掛け合わせる」:
 * Q and K are rotated by position after the projections; the standard rotary
 * form, see retention_rope).  The rotated copies live in the workspace, so
 * the caller keeps q and k unrotated and needs no buffers of its own.
 * Schedule: one rotary pass over q and k, then the two chunkwise passes.
 * (Rotating k inside the state pass instead was measured slower on B200: the
 * angle reduction lands on the converter warps that set the state pass's
 * pace.)
 * Arguments as retention_chunkwise_fwd, plus rope_base (> 1, finite); bf16
 * inputs only (RET_ERR_UNSUPPORTED otherwise), dk even.  q and k are not
 * modified.  workspace: at least retention_chunkwise_fwd_rope_workspace_size()
 * bytes, 256-byte aligned (it holds the chunkwise workspace, then the rotated
 * q and k).
 */
RET_API size_t retention_chunkwise_fwd_rope_workspace_size(int chunk, int B, int T, int H,
                                                            int dk, int dv, int nseq);
RET_API ret_status retention_chunkwise_fwd_rope(const void* q, const void* k, const void* v,
                                                ret_dtype in_dtype, const double* gamma,
                                                int chunk, const int32_t* cu_seqlens, int nseq,
                                                const float* state_in, float* state_out,
                                                void* out, ret_dtype out_dtype,
                                                const ret_norm_gate* ng, double rope_base,
                                                void* workspace, size_t workspace_bytes,
                                                int B, int T, int H, int dk, int dv,
                                                ret_stream_t stream);

/*
 * Standalone per-head GroupNorm + Swish gate (the epilogue that
 * retention_chunkwise_fwd fuses when given `ng`).
 *   o: [ntok, H, dv] o_dtype     y: [ntok, H, dv] y_dtype (may not alias o)
 *   ng: gate, optional affine and eps as in ret_norm_gate (required).
 * Supported: dv in 1..1024.
 */
RET_API ret_status msr_norm_gate(const void* o, ret_dtype o_dtype, const ret_norm_gate* ng,
                         void* y, ret_dtype y_dtype, int ntok, int H, int dv,
                         ret_stream_t stream);

/*
 * Synchronises `stream`, then reads and clears this device's error word, which
 * the kernels set instead of trapping: RET_ERR_TIMEOUT when a bounded
 * wait inside a kernel gave up (the kernel then skipped its remaining work
 * and released what it held), RET_ERR_DEVICE_DATA when cu_seqlens was
 * inconsistent, RET_ERR_RANGE when a tensor-core operand left fp16's range
 * (the outputs of that call are then not reliable).  Returns RET_OK when no such event happened since the last
 * call, RET_ERR_CUDA if the synchronisation itself failed.
 */
RET_API ret_status retention_check_device_error(ret_stream_t stream);

/*
 * Failure-detection self-test (no counterpart on the pages: it exercises this
 * library's own time-out path).  Enqueues on `stream` one single-warp kernel
 * that waits on a shared-memory barrier nothing ever arrives on, through the
 * same bounded wait every tensor-core kernel uses (about 2 s of SM clock).
 * When the bound expires the kernel sets the device error word and returns,
 * so a following retention_check_device_error() returns RET_ERR_TIMEOUT and
 * the context stays usable.  Returns RET_ERR_CUDA if the launch failed.
 */
RET_API ret_status retention_selftest_wait_timeout(ret_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* RETENTION_H_ */
