/*
 * kda.h -- C ABI of the B200 (sm_100a) Kimi Delta Attention (KDA) library.
 *
 * KDA is the gated delta rule with a per-channel gate.  For every sequence and
 * head the library carries a state S (d_k x d_v, fp32) and, for each token t
 * with query q_t, key k_t (d_k), value v_t (d_v), per-channel log decay
 * log_alpha_t (d_k) and write rate beta_t (scalar), computes
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T q_t
 *
 * i.e. decay the old state channel by channel, read the old answer with the
 * key, form the error against v_t, write beta_t times the error back along the
 * key, then read the output with the query.
 *
 * Where the operation is defined (web pages, cited by title / address):
 *   - delta rule S <- S + k^T (v - S k) and the scalar gate alpha in [0, 1]
 *     (alpha = 1: pure delta rule, alpha = 0: memory cleared):
 *     "From GPT-2 to Kimi K3" essay, pwwt.cn/news/3716252, delta-rule and
 *     Gated DeltaNet paragraphs;
 *   - one alpha per channel instead of one per head: same essay, Kimi Linear
 *     paragraph; "我终于看懂了 KDA" explainer, pwwt.cn/news/3787313, section 9;
 *   - order decay -> read -> error -> write and the learning rate beta:
 *     the explainer, sections 6 and 8;
 *   - chunkwise prefill (chunk C = 64 or 128, masked attention inside a chunk,
 *     state-first recurrence across chunks) with WY / DPLR restructuring:
 *     the essay's chunkwise paragraph; the explainer, sections 16 and 17;
 *   - token-by-token decode (read state, emit output, update state):
 *     the explainer, section 15.
 *
 * Conventions shared by all calls
 *   - Device pointers are caller-owned CUDA device memory; the library keeps no
 *     reference after a call returns and never allocates device memory.
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*; NULL is
 *     the legacy default stream).  Input validation happens on the host before
 *     anything is launched: a call that returns an error other than
 *     KDA_ERR_CUDA has launched nothing and written nothing.
 *   - Token-major layouts, last dimension contiguous:
 *       q, k, log_alpha : [B, T, H, dk]      v, o : [B, T, H, dv]
 *       beta            : [B, T, H]
 *       states          : [N, H, dk, dv] fp32 (dv contiguous)
 *     For packed variable-length batches B = 1, T = total tokens, and
 *     cu_seqlens gives the N + 1 sequence offsets.
 *   - q, k, v, log_alpha, beta and o share one dtype (KDA_BF16 or KDA_F32);
 *     states are always fp32; accumulation is fp32.
 *   - log_alpha <= 0 (alpha in [0, 1]); -inf means alpha = 0.  Kernels clamp
 *     log_alpha at -100 (exp(-100) is below every fp32 normal number).
 *   - No scaling of q is applied: o_t = S_t^T q_t exactly.
 *   - Supported sizes: dk, dv in {64, 128}; every pointer 16-byte aligned.
 */
#ifndef KDA_H_
#define KDA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KDA_API __attribute__((visibility("default")))
#else
#define KDA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    KDA_OK = 0,
    KDA_ERR_NULL = -1,       /* a required pointer is NULL                     */
    KDA_ERR_SHAPE = -2,      /* unsupported or inconsistent sizes              */
    KDA_ERR_DTYPE = -3,      /* unknown dtype                                  */
    KDA_ERR_ALIGN = -4,      /* a pointer is not 16-byte aligned               */
    KDA_ERR_CHUNK = -5,      /* chunk size is not 64 or 128                    */
    KDA_ERR_SEQLENS = -6,    /* cu_seqlens not 0-based, non-decreasing, = T    */
    KDA_ERR_WORKSPACE = -7,  /* workspace NULL or smaller than required        */
    KDA_ERR_CUDA = -8,       /* a CUDA runtime call or launch failed           */
    KDA_ERR_TIMEOUT = -9,    /* a bounded device-side wait gave up             */
    KDA_ERR_DEVICE = -10,    /* the current device is not sm_100 (B200)       */
    KDA_ERR_SCRATCH = -11    /* problem too large for the built-in scratch     */
} kda_status;

typedef enum {
    KDA_BF16 = 0,
    KDA_F32 = 1
} kda_dtype;

/* Prefill algorithm.  AUTO picks the tensor-core path for bf16 with
 * dk = dv = 128 and the CUDA-core path otherwise.  SIMT is the four-kernel
 * CUDA-core split (cumulative decay, WY/UT, state carry, output) that keeps
 * its intermediates in the workspace; TC is the tcgen05 tensor-core path. */
typedef enum {
    KDA_ALGO_AUTO = 0,
    KDA_ALGO_SIMT = 1,
    KDA_ALGO_TC = 2
} kda_algo;

/* Human-readable name of a status code (static string, never NULL). */
KDA_API const char* kda_status_string(int status);

/* Library version as 10000 * major + 100 * minor + patch. */
KDA_API int kda_version(void);

/*
 * Workspace bytes kda_chunk_fwd needs for this problem (0 on invalid sizes).
 *   cu_seqlens_host : NULL for B sequences of length T each; else a HOST array of
 *                     n_seqs + 1 int32 offsets (requires B == 1).
 */
KDA_API size_t kda_chunk_fwd_workspace_size(int B, int T, int H, int dk, int dv, int C,
                                    kda_dtype dtype, const int32_t* cu_seqlens_host,
                                    int n_seqs);

/* As above for a chosen algorithm (AUTO resolves as kda_chunk_fwd does). */
KDA_API size_t kda_chunk_fwd_workspace_size_ex(int B, int T, int H, int dk, int dv, int C,
                                       kda_dtype dtype, const int32_t* cu_seqlens_host,
                                       int n_seqs, kda_algo algo);

/*
 * Chunkwise prefill.  Processes every sequence from its initial state and
 * writes o for every token and (optionally) the final state of every sequence.
 *
 *   q, k, v, log_alpha, beta : device inputs (layouts above), dtype `dtype`
 *   init_state      : device [N, H, dk, dv] fp32, or NULL for zero states
 *   cu_seqlens_host : NULL (B sequences of T tokens) or a HOST array of
 *                     n_seqs + 1 int32 offsets, cu[0] = 0, non-decreasing,
 *                     cu[n_seqs] = T, with B = 1; empty sequences are allowed
 *   n_seqs          : number of sequences when cu_seqlens_host != NULL
 *   C               : chunk size, 64 or 128; chunks restart at each sequence
 *                     start and the last chunk of a sequence may be partial.
 *                     The chunk form's result does not depend on C (up to
 *                     rounding), so the tensor-core path serves both sizes with
 *                     64-token chunks; the CUDA-core path uses C as given
 *   o               : device output [B, T, H, dv], dtype `dtype`
 *   final_state     : device [N, H, dk, dv] fp32, or NULL; may alias init_state
 *   workspace       : device scratch of at least kda_chunk_fwd_workspace_size()
 *                     bytes, 256-byte aligned; contents on entry are ignored
 *   stream          : cudaStream_t (as void*)
 * T == 0 (or all sequences empty) is valid: final_state = init_state (or 0).
 */
KDA_API kda_status kda_chunk_fwd(const void* q, const void* k, const void* v,
                         const void* log_alpha, const void* beta, kda_dtype dtype,
                         const float* init_state, const int32_t* cu_seqlens_host,
                         int n_seqs, int B, int T, int H, int dk, int dv, int C,
                         void* o, float* final_state, void* workspace,
                         size_t workspace_bytes, void* stream);

/* kda_chunk_fwd with an explicit algorithm choice (same arguments otherwise). */
KDA_API kda_status kda_chunk_fwd_ex(const void* q, const void* k, const void* v,
                            const void* log_alpha, const void* beta, kda_dtype dtype,
                            const float* init_state, const int32_t* cu_seqlens_host,
                            int n_seqs, int B, int T, int H, int dk, int dv, int C,
                            void* o, float* final_state, void* workspace,
                            size_t workspace_bytes, void* stream, kda_algo algo);

/*
 * Prefill of a packed batch held in HOST memory, with the transfers overlapped
 * with the computation.  The sequences are taken in `n_groups` groups of
 * consecutive sequences with about equal token counts; while group g is
 * computed (on `stream`), group g + 1's inputs are copied to the device and
 * group g - 1's outputs back to the host, on two streams of the library's own,
 * so that both copy directions and the kernels run at once.  Each group is one
 * kda_chunk_fwd call on device staging inside `device_buffer`, so every output
 * equals, bit for bit, the device call's on the whole batch (a sequence's
 * result does not depend on the other sequences).  This is the library's
 * transfer pipeline around the operation, not part of the pages' method.
 *
 *   q, k, v, log_alpha, beta : HOST inputs, layouts as kda_chunk_fwd with B = 1;
 *                     page-locked memory (cudaHostAlloc / cudaHostRegister) lets
 *                     the copies overlap; pageable memory works, serialised
 *   init_state      : HOST [N, H, dk, dv] fp32, or NULL for zero states
 *   cu_seqlens_host : HOST n_seqs + 1 int32 offsets (as kda_chunk_fwd; required)
 *   o               : HOST output [1, T, H, dv], dtype `dtype`
 *   final_state     : HOST [N, H, dk, dv] fp32, or NULL
 *   n_groups        : >= 1; more groups overlap more but each call costs a
 *                     launch sequence (8 suits batches of ~10^6 tokens); values
 *                     above n_seqs act as n_seqs
 *   device_buffer   : device scratch of kda_chunk_fwd_host_buffer_size() bytes
 *                     (same sizes and n_groups), 256-byte aligned; ownership
 *                     stays with the caller, contents on entry are ignored
 *   stream          : cudaStream_t (as void*): the call's work starts after the
 *                     work already on `stream`, and `stream` waits for all of it
 *                     (copies back included); the call returns without waiting,
 *                     so the host buffers must stay valid until `stream` is done
 * Errors: as kda_chunk_fwd (KDA_ERR_SEQLENS for a NULL cu_seqlens_host,
 * KDA_ERR_WORKSPACE for a short device_buffer), KDA_ERR_CUDA if a stream, event
 * or copy cannot be made.  A bounded device wait that expired in any group is
 * reported by kda_chunk_fwd_host_device_status.
 */
KDA_API size_t kda_chunk_fwd_host_buffer_size(kda_dtype dtype, const int32_t* cu_seqlens_host, int n_seqs,
                                              int H, int dk, int dv, int C, int n_groups);
KDA_API kda_status kda_chunk_fwd_host(const void* q, const void* k, const void* v, const void* log_alpha,
                                      const void* beta, kda_dtype dtype, const float* init_state,
                                      const int32_t* cu_seqlens_host, int n_seqs, int H, int dk, int dv,
                                      int C, void* o, float* final_state, int n_groups, void* device_buffer,
                                      size_t device_buffer_bytes, void* stream);
/* Synchronises `stream`; KDA_OK, or the first error a group's kernels recorded
 * (KDA_ERR_TIMEOUT) in the last kda_chunk_fwd_host call that used device_buffer. */
KDA_API kda_status kda_chunk_fwd_host_device_status(const void* device_buffer, void* stream);

/*
 * Byte offsets, inside the workspace of the SIMT algorithm, of the
 * intermediates that its four kernels exchange (for inspection by tests):
 *   offsets[0] g       fp32 [T_total, H, dk]  chunk-local inclusive cumulative log decay
 *   offsets[1] U       fp32 [T_total, H, dv]  (I + A)^-1 Diag(beta) V
 *   offsets[2] Wk      fp32 [T_total, H, dk]  (I + A)^-1 Diag(beta) (K . exp(g))
 *   offsets[3] W       fp32 [T_total, H, dv]  per-token corrections U - Wk S_n
 *   offsets[4] S_chunk fp32 [n_chunks, H, dk, dv] start state of every chunk
 * (T_total = B * T; chunks are numbered sequence by sequence.)  Same size
 * arguments as kda_chunk_fwd_workspace_size.
 */
KDA_API kda_status kda_chunk_simt_offsets(int B, int T, int H, int dk, int dv, int C,
                                  const int32_t* cu_seqlens_host, int n_seqs,
                                  size_t offsets[5]);

/*
 * Optional per-kernel timing hook for the calling host thread.  When n_events
 * > 0, the next kda_chunk_fwd / kda_chunk_fwd_ex call made from this thread
 * records events[0] on its stream before its first kernel and events[i] after
 * its i-th kernel (i = 1 .. number of kernels), then clears the hook.  Calls
 * that launch more kernels than n_events - 1 record only the first ones.
 *   events   : array of cudaEvent_t (as void*), created by the caller
 *   n_events : number of entries (0 clears the hook)
 * The events only observe the launches; kda_chunk_fwd_kernels tells how many
 * kernels a call launches and their names.
 */
KDA_API kda_status kda_set_timing_events(void* const* events, int n_events);

/*
 * Test hook for the failure path of the bounded device-side waits (no
 * counterpart on the pages; it exists so that tests can make a wait expire
 * without breaking anything on the GPU).  Arms, for the next tensor-core
 * prefill (kda_chunk_fwd / _ex / _prep / _noalloc) called from this host
 * thread, one extra wait in the first CTA of the chosen kernels on a barrier
 * that nothing ever completes, bounded by limit_ns.  That wait expires: the
 * kernel records KDA_ERR_TIMEOUT (read back with kda_chunk_fwd_device_status),
 * waits for the copies and products it has already issued, frees its tensor
 * memory and returns; the call's outputs are then undefined.  The next call is
 * unaffected.
 *   kernels  : bit 0 the chunk-local kernel (tc_intra), bit 1 the state carry
 *              (tc_recur); 0 disarms
 *   limit_ns : 1 .. 1e9 (ignored when kernels == 0)
 * Errors: KDA_ERR_SHAPE for unknown bits or a limit out of range.
 */
KDA_API kda_status kda_set_test_wait_limit(unsigned int kernels, unsigned long long limit_ns);

/*
 * Number of kernels kda_chunk_fwd_ex launches for this problem and algorithm
 * (after AUTO resolution), and their names through names[i] (static strings;
 * names may be NULL, at most max_names entries are written).  Returns the
 * count, or a negative kda_status on invalid sizes.
 */
KDA_API int kda_chunk_fwd_kernels(int B, int T, int H, int dk, int dv, int C, kda_dtype dtype,
                                  const int32_t* cu_seqlens_host, int n_seqs, kda_algo algo,
                                  const char** names, int max_names);

/*
 * Prefill that allocates nothing (no counterpart on the pages: this is a
 * deployment aid, not part of the method).
 *
 * For callers that cannot allocate device memory -- a plugin host that passes
 * the operator only its input and output buffers and no allocator, or a
 * serving runtime whose memory pool already owns the whole device, where a
 * cudaMalloc from inside the operator fails or forces a device-wide
 * synchronisation.  Same arguments and results as kda_chunk_fwd, without the
 * workspace: the scratch is a fixed array of KDA_NOALLOC_SCRATCH_BYTES in
 * device memory that the library itself declares.  Every device that loads the
 * library holds that array until the process exits.
 *
 *   - A problem fits exactly when kda_chunk_fwd_workspace_size() <=
 *     KDA_NOALLOC_SCRATCH_BYTES; larger ones are rejected with KDA_ERR_SCRATCH
 *     before anything is launched.  From the scratch layouts: the tensor-core
 *     path (bf16, dk = dv = 128) needs 147,968 bytes per (64-token chunk, head),
 *     about 450 chunk-heads (e.g. B = 1, T = 1792, H = 16); the CUDA-core path
 *     needs 4 (3 dk + 2 dv) bytes per token-head plus 4 dk dv bytes per
 *     (chunk, head), about 18.7 K token-heads at dk = dv = 128, C = 64 and about
 *     43 K at dk = dv = 64, C = 64; packed batches add 32 bytes per sequence.
 *   - The call never calls cudaMalloc, cudaFree or any allocating routine.
 *   - The first call on a device looks up the array's device address with that
 *     device current (cudaGetSymbolAddress) and caches it for the process; make
 *     that first call before any stream capture on the device.  Destroying the
 *     device's primary context between calls (cudaDeviceReset) is not
 *     supported: the cached address would no longer be valid.
 *   - All calls share the one array, and it keeps the last call's contents
 *     (the prefill writes every scratch byte before reading it, so nothing needs
 *     clearing).  Calls whose execution overlaps on the GPU -- on different
 *     streams, or from different host threads -- race on the array and give
 *     wrong results: serialise them.
 */
#define KDA_NOALLOC_SCRATCH_BYTES (64u << 20)

KDA_API kda_status kda_chunk_fwd_noalloc(const void* q, const void* k, const void* v,
                                         const void* log_alpha, const void* beta, kda_dtype dtype,
                                         const float* init_state, const int32_t* cu_seqlens_host,
                                         int n_seqs, int B, int T, int H, int dk, int dv, int C,
                                         void* o, float* final_state, void* stream);

/*
 * One decode step for N independent sequences, one token each; the state is
 * updated in place (read once, written once).
 *   q, k, log_alpha : device [N, H, dk]; v : device [N, H, dv]; beta : [N, H]
 *   state           : device [N, H, dk, dv] fp32, read and overwritten
 *   o               : device [N, H, dv], dtype `dtype`
 */
KDA_API kda_status kda_decode_step(const void* q, const void* k, const void* v,
                           const void* log_alpha, const void* beta, kda_dtype dtype,
                           float* state, int N, int H, int dk, int dv, void* o,
                           void* stream);

/*
 * Input preprocessing fused into the kernels (the gate and the key/query
 * normalisation that usually run as separate passes before the operator).
 * The per-channel decay comes from an "alpha projection" with alpha between 0
 * and 1 ("22580倍参数量级" article, tahou.com/article/213680821660188677,
 * sections on Gated DeltaNet and on the Kimi Linear architecture), but the pages
 * do not fix the gate's parametrisation; this library reads it as
 *   KDA_PREP_QK_L2NORM     : q and k are divided by their L2 norm over d_k
 *                            (per token and head; an all-zero vector stays 0)
 *   KDA_PREP_GATE_SOFTPLUS : the log_alpha argument holds raw gate logits a,
 *                            log alpha = -softplus(a) = -log(1 + e^a)
 *   KDA_PREP_BETA_SIGMOID  : the beta argument holds raw logits b,
 *                            beta = 1 / (1 + e^-b)
 * Flags combine with |.  With no flag the calls below are kda_chunk_fwd and
 * kda_decode_step.
 */
typedef enum {
    KDA_PREP_NONE = 0,
    KDA_PREP_QK_L2NORM = 1,
    KDA_PREP_GATE_SOFTPLUS = 2,
    KDA_PREP_BETA_SIGMOID = 4
} kda_prep;

/*
 * kda_chunk_fwd with the inputs preprocessed inside the tensor-core kernels
 * (same arguments, layouts, workspace and errors; `prep` is a kda_prep mask).
 * The preprocessing is fused into the tensor-core path only: with prep != 0,
 * problems that path does not take (fp32, dk or dv of 64) are rejected with
 * KDA_ERR_SHAPE, as is a mask with unknown bits.
 */
KDA_API kda_status kda_chunk_fwd_prep(const void* q, const void* k, const void* v,
                                      const void* log_alpha, const void* beta, kda_dtype dtype,
                                      unsigned int prep, const float* init_state,
                                      const int32_t* cu_seqlens_host, int n_seqs,
                                      int B, int T, int H, int dk, int dv, int C,
                                      void* o, float* final_state,
                                      void* workspace, size_t workspace_bytes, void* stream);

/* kda_decode_step with the inputs preprocessed inside the decode kernel (all
 * shapes and dtypes of kda_decode_step; unknown bits: KDA_ERR_SHAPE). */
KDA_API kda_status kda_decode_step_prep(const void* q, const void* k, const void* v,
                                        const void* log_alpha, const void* beta, kda_dtype dtype,
                                        unsigned int prep, float* state, int N, int H, int dk, int dv,
                                        void* o, void* stream);


/*
 * Chunkwise backward pass (training): the gradients of
 *   L = sum(d_o * o) + sum(d_final_state * final_state)
 * where o and final_state are what kda_chunk_fwd computes from the same
 * inputs.  The pages say training needs the chunkwise parallel form ("From
 * GPT-2 to Kimi K3" essay, pwwt.cn/news/3716252, chunkwise paragraph) but
 * derive no backward pass; this one is the chain rule applied to that form.
 *
 *   q, k, v, log_alpha, beta, init_state, cu_seqlens_host, n_seqs, B, T, H,
 *   dk, dv, C       : the forward call's arguments (same meaning and layout)
 *   d_o             : device [B, T, H, dv], dtype `dtype`
 *   d_final_state   : device [N, H, dk, dv] fp32, or NULL (zero)
 *   dq, dk, dlog_alpha : device [B, T, H, dk], dtype `dtype` (written)
 *   dv              : device [B, T, H, dv], dtype `dtype` (written)
 *   dbeta           : device [B, T, H], dtype `dtype` (written)
 *   d_init_state    : device [N, H, dk, dv] fp32, or NULL (not written); the
 *                     gradient for init_state (for a zero initial state when
 *                     init_state is NULL)
 *   workspace       : >= kda_chunk_bwd_workspace_size(...) bytes, 256-byte
 *                     aligned, caller-owned, not read before it is written
 *
 * The forward intermediates are recomputed inside the call, with 64-token
 * chunks whatever C asks for (the chunk form does not depend on the chunk
 * length): by the tensor-core forward for bf16 with dk = dv = 128, by the
 * fp32 CUDA-core kernels otherwise; the gradient kernels run in fp32.  dlog_alpha is zero where log_alpha is below
 * the kernels' floor of -100 (log alpha = -inf included).  dlog_alpha and dk
 * add per-tile contributions with shared-memory atomics, so repeated calls may
 * differ in their last bits; dq, dv, dbeta and d_init_state are reproducible.  Errors as
 * kda_chunk_fwd; all output pointers must be distinct from the inputs.
 */
KDA_API size_t kda_chunk_bwd_workspace_size(int B, int T, int H, int dk, int dv, int C,
                                            const int32_t* cu_seqlens_host, int n_seqs);

KDA_API kda_status kda_chunk_bwd(const void* q, const void* k, const void* v,
                                 const void* log_alpha, const void* beta, kda_dtype dtype,
                                 const float* init_state, const int32_t* cu_seqlens_host,
                                 int n_seqs, int B, int T, int H, int dk, int dv, int C,
                                 const void* d_o, const float* d_final_state,
                                 void* dq, void* dk_out, void* dv_out, void* dlog_alpha,
                                 void* dbeta, float* d_init_state,
                                 void* workspace, size_t workspace_bytes, void* stream);


/*
 * One sequence split over several devices: the affine map of a segment.
 *
 * The state carried from chunk to chunk ("From GPT-2 to Kimi K3" essay,
 * pwwt.cn/news/3716252, chunkwise paragraph) depends affinely on the state a
 * segment of tokens starts from: for every sequence and head the segment maps
 * its start state S to
 *     S_end = M S + F,
 * M (d_k x d_k) being the segment's final state from the identity with the
 * values' contribution left out, and F (d_k x d_v) its final state from a zero
 * start.  A device holding a later segment computes (M, F) of its own segment
 * in one pass, the maps are exchanged (one all-gather), each device chains the
 * maps of the segments before it (kda_compose_states) and runs kda_chunk_fwd
 * from the start state that gives.  (The split is this library's construction,
 * not a step the pages describe.)
 *
 *   q, k, v, log_alpha, beta, dtype, cu_seqlens_host, n_seqs, B, T, H, dk,
 *   dv, C            : as kda_chunk_fwd (no initial state: it does not enter
 *                      the map)
 *   M                : device [N, H, dk, dk] fp32 (written)
 *   F                : device [N, H, dk, dv] fp32 (written)
 *   workspace        : >= kda_chunk_fwd_workspace_size(...) bytes, as for
 *                      kda_chunk_fwd
 * Errors as kda_chunk_fwd.  Asynchronous on `stream`.  M equals the identity
 * and F zero for an empty sequence.
 */
KDA_API kda_status kda_chunk_segment_map(const void* q, const void* k, const void* v, const void* log_alpha,
                                         const void* beta, kda_dtype dtype, const int32_t* cu_seqlens_host,
                                         int n_seqs, int B, int T, int H, int dk, int dv, int C, float* M, float* F,
                                         void* workspace, size_t workspace_bytes, void* stream);

/*
 * Start states of R consecutive segments chained through their maps:
 *     states[0] = init_state (or zero),  states[r + 1] = M_r states[r] + F_r
 * for r = 0 .. R - 1, fp32 on the device.
 *   M          : device [R, N, H, dk, dk] fp32 (kda_chunk_segment_map's M of each segment)
 *   F          : device [R, N, H, dk, dv] fp32
 *   init_state : device [N, H, dk, dv] fp32, or NULL for zero
 *   states     : device [R + 1, N, H, dk, dv] fp32 (written; may not alias M, F or init_state)
 * R = 0 copies init_state (or zero) to states[0].  Errors: KDA_ERR_SHAPE (sizes),
 * KDA_ERR_NULL, KDA_ERR_ALIGN (16 bytes), KDA_ERR_CUDA.  Asynchronous on `stream`.
 */
KDA_API kda_status kda_compose_states(const float* M, const float* F, const float* init_state, int R, int N, int H,
                                      int dk, int dv, float* states, void* stream);

/*
 * Device-side status of a finished call.  The tensor-core kernels bound every
 * wait on the device (2 s); if one expires they stop, leave their outputs
 * undefined and record KDA_ERR_TIMEOUT in an error word inside the workspace
 * (cleared at the start of each call).  These two calls synchronise `stream`
 * and return KDA_OK or the recorded error for the last kda_chunk_fwd[_ex|_prep]
 * / kda_chunk_bwd call that used `workspace` with the same size arguments.
 * They copy 4 bytes of the caller-owned workspace to the host and write
 * nothing.  (No counterpart on the pages: this is part of the library's
 * failure handling, not of the operation.)
 * For problems on the CUDA-core path they return KDA_OK without touching the
 * device (those kernels do not wait on the device).  Errors: KDA_ERR_NULL for a
 * NULL workspace, the size errors of the calls themselves, KDA_ERR_CUDA if the
 * copy or the synchronisation fails.
 */
KDA_API kda_status kda_chunk_fwd_device_status(const void* workspace, kda_dtype dtype,
                                               const int32_t* cu_seqlens_host, int n_seqs,
                                               int B, int T, int H, int dk, int dv, int C,
                                               kda_algo algo, void* stream);
KDA_API kda_status kda_chunk_bwd_device_status(const void* workspace, kda_dtype dtype,
                                               const int32_t* cu_seqlens_host, int n_seqs,
                                               int B, int T, int H, int dk, int dv, int C,
                                               void* stream);
/* The same for the last kda_chunk_fwd_noalloc call on the current device
 * (its scratch is the library's own array). */
KDA_API kda_status kda_chunk_fwd_noalloc_device_status(kda_dtype dtype, const int32_t* cu_seqlens_host,
                                                       int n_seqs, int B, int T, int H, int dk, int dv,
                                                       int C, void* stream);


#ifdef __cplusplus
}
#endif

#endif /* KDA_H_ */
