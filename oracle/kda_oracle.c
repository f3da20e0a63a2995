/*
 * KDA reference oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, fp64 CPU implementation of the Kimi Delta Attention (KDA)
 * recurrence.  Only the test-suite, the smoke check and the CPU-baseline leg
 * of the benchmark may load this file.  It shares no code, header, table or
 * helper with the CUDA library, and the CUDA library never loads it.
 *
 * Sources (web pages, cited by title / address and section):
 *   [ESSAY]   "From GPT-2 to Kimi K3" essay, pwwt.cn/news/3716252
 *             - delta-rule paragraph: S <- S + k^T (v - S k)
 *             - Gated DeltaNet paragraph: alpha in [0,1] decays the previous
 *               state; alpha = 1 gives the delta rule, alpha = 0 clears memory
 *             - Kimi Linear paragraph: every channel has its own alpha
 *             - chunkwise paragraph: chunks of size C, masked attention inside
 *               a chunk, state-first recurrence across chunks, C = 1 is the
 *               token recurrence
 *   [EXPLAIN] "我终于看懂了 KDA" explainer, pwwt.cn/news/3787313
 *             - section 6 (delta rule): read the old value with the key, form
 *               the error, write learning_rate * error back along the key
 *             - section 8 (forgetting): decay the old state with the gate,
 *               then read with the current key, then compute the error, then
 *               write the correction
 *             - section 9 (fine-grained gate): per-channel decay
 *             - sections 16-17 (chunkwise, WY / DPLR): recurrent across
 *               chunks, parallel inside a chunk
 *
 * Reading adopted where the pages leave the step open:
 *   - state S is d_k x d_v per head; alpha decays the key dimension (rows);
 *     the read is S^T k and the output is o_t = S_t^T q_t (after the write)
 *   - beta (the "learning rate") is one scalar per (token, head)
 *   - log_alpha = -inf means alpha = 0 exactly
 *
 * Data layout (all fp64, row-major, last dimension contiguous):
 *   q, k, log_alpha : [n_tokens, H, dk]
 *   v               : [n_tokens, H, dv]
 *   beta            : [n_tokens, H]
 *   seq_start       : [n_seqs + 1] token offsets, seq_start[0] = 0
 *   init_state      : [n_seqs, H, dk, dv] or NULL (zero state)
 *   o               : [n_tokens, H, dv]            (output)
 *   final_state     : [n_seqs, H, dk, dv] or NULL  (output)
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------
 * O1: token-by-token recurrence, the definition.
 *
 * For each sequence and head, independently:
 *   S <- init_state (or 0)
 *   for each token t in order:
 *     S[c,:] <- alpha_t[c] * S[c,:]          decay first      [EXPLAIN s8, s9]
 *     r      <- S^T k_t                      read old answer  [EXPLAIN s6]
 *     u      <- v_t - r                      error            [EXPLAIN s6]
 *     S      <- S + beta_t * k_t u^T         write correction [ESSAY delta rule]
 *     o_t    <- S^T q_t                      read after write
 *   final_state <- S
 * The (seq, head) pairs are independent; they are spread over threads, which
 * does not change any arithmetic.
 * ---------------------------------------------------------------------- */
int kda_ref_forward_f64(const double* q, const double* k, const double* v,
                        const double* log_alpha, const double* beta,
                        const double* init_state, const int64_t* seq_start,
                        int n_seqs, int H, int dk, int dv,
                        double* o, double* final_state, int n_threads)
{
    if (n_seqs < 0 || H <= 0 || dk <= 0 || dv <= 0) return -1;
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#else
    (void)n_threads;
#endif
    long n_pairs = (long)n_seqs * H;
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (long p = 0; p < n_pairs; ++p) {
        int n = (int)(p / H), h = (int)(p % H);
        double* S = (double*)malloc(sizeof(double) * (size_t)dk * dv);
        double* r = (double*)malloc(sizeof(double) * (size_t)dv);
        double* a = (double*)malloc(sizeof(double) * (size_t)dk);
        if (!S || !r || !a) {
            free(S); free(r); free(a);
#pragma omp atomic write
            failed = 1;
            continue;
        }
        if (init_state)
            memcpy(S, init_state + ((size_t)n * H + h) * dk * dv, sizeof(double) * (size_t)dk * dv);
        else
            memset(S, 0, sizeof(double) * (size_t)dk * dv);

        for (int64_t t = seq_start[n]; t < seq_start[n + 1]; ++t) {
            const double* qt = q + ((size_t)t * H + h) * dk;
            const double* kt = k + ((size_t)t * H + h) * dk;
            const double* vt = v + ((size_t)t * H + h) * dv;
            const double* lat = log_alpha + ((size_t)t * H + h) * dk;
            double bt = beta[(size_t)t * H + h];
            double* ot = o + ((size_t)t * H + h) * dv;

            /* decay: alpha = exp(log_alpha); exp(-inf) = 0 exactly */
            for (int c = 0; c < dk; ++c) a[c] = exp(lat[c]);
            for (int c = 0; c < dk; ++c)
                for (int j = 0; j < dv; ++j) S[(size_t)c * dv + j] *= a[c];
            /* read the old answer with the key: r = S^T k */
            for (int j = 0; j < dv; ++j) r[j] = 0.0;
            for (int c = 0; c < dk; ++c)
                for (int j = 0; j < dv; ++j) r[j] += S[(size_t)c * dv + j] * kt[c];
            /* error u = v - r, written back along the key with rate beta */
            for (int c = 0; c < dk; ++c)
                for (int j = 0; j < dv; ++j)
                    S[(size_t)c * dv + j] += bt * kt[c] * (vt[j] - r[j]);
            /* output o = S^T q with the updated state */
            for (int j = 0; j < dv; ++j) ot[j] = 0.0;
            for (int c = 0; c < dk; ++c)
                for (int j = 0; j < dv; ++j) ot[j] += S[(size_t)c * dv + j] * qt[c];
        }
        if (final_state)
            memcpy(final_state + ((size_t)n * H + h) * dk * dv, S, sizeof(double) * (size_t)dk * dv);
        free(S); free(r); free(a);
    }
    return failed ? -2 : 0;
}

/* ------------------------------------------------------------------------
 * O2: brute chunk form (chunk size C >= 1, any C, including C >= length).
 *
 * Each sequence is cut into chunks of C consecutive tokens starting at the
 * sequence start (the last one may be shorter) [EXPLAIN s16].  Inside a chunk
 * with start state S0 and rows r = 0..L-1 (all products over channels c are
 * elementwise, alpha = exp(log_alpha)):
 *   Gam_r[c]    = prod_{j<=r} alpha_j[c]                (decay from chunk start)
 *   D(r,i)[c]   = prod_{i<j<=r} alpha_j[c]              (pairwise decay, i <= r)
 *   A[r,i]      = beta_r * sum_c k_r[c] k_i[c] D(r,i)[c]          (i < r)
 *   (I + A) U   = Diag(beta) V                          (WY / UT form)
 *   (I + A) Wk  = Diag(beta) (K . Gam)
 *   W           = U - Wk S0            (the per-token corrections beta*u)
 *   O[r]        = S0^T (Gam_r . q_r) + sum_{i<=r} (sum_c q_r[c] k_i[c] D(r,i)[c]) W[i]
 *   S_next      = Diag(Gam_{L-1}) S0 + sum_i (k_i . D(L-1,i)) W[i]^T
 * The decays are formed as plain products of alpha (never as a difference of
 * cumulative logs), so alpha = 0 and any decay range are handled exactly.
 * The triangular systems are solved by forward substitution, row by row.
 *
 * Optional intermediate outputs (pass NULL to skip), laid out per chunk in
 * the global chunk order (sequence by sequence, chunk by chunk, head fastest):
 *   g_out     [n_tokens, H, dk]  inclusive chunk-local cumulative log decay
 *   u_out     [n_tokens, H, dv]  U rows
 *   wk_out    [n_tokens, H, dk]  Wk rows
 *   w_out     [n_tokens, H, dv]  W rows
 *   s_chunk   [n_chunks_total, H, dk, dv]  start state of every chunk
 * ---------------------------------------------------------------------- */
int kda_ref_chunkform_f64(const double* q, const double* k, const double* v,
                          const double* log_alpha, const double* beta,
                          const double* init_state, const int64_t* seq_start,
                          int n_seqs, int H, int dk, int dv, int C,
                          double* o, double* final_state,
                          double* g_out, double* u_out, double* wk_out,
                          double* w_out, double* s_chunk, int n_threads)
{
    if (n_seqs < 0 || H <= 0 || dk <= 0 || dv <= 0 || C <= 0) return -1;
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#else
    (void)n_threads;
#endif
    /* first chunk index of each sequence, for s_chunk */
    int64_t* chunk_base = (int64_t*)malloc(sizeof(int64_t) * (size_t)(n_seqs + 1));
    if (!chunk_base) return -2;
    chunk_base[0] = 0;
    for (int n = 0; n < n_seqs; ++n) {
        int64_t len = seq_start[n + 1] - seq_start[n];
        chunk_base[n + 1] = chunk_base[n] + (len + C - 1) / C;
    }
    long n_pairs = (long)n_seqs * H;
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (long p = 0; p < n_pairs; ++p) {
        int n = (int)(p / H), h = (int)(p % H);
        size_t sz = (size_t)dk * dv;
        double* S0 = (double*)malloc(sizeof(double) * sz);
        double* Snext = (double*)malloc(sizeof(double) * sz);
        double* Gam = (double*)malloc(sizeof(double) * (size_t)C * dk);
        double* D = (double*)malloc(sizeof(double) * (size_t)C * C * dk);
        double* A = (double*)malloc(sizeof(double) * (size_t)C * C);
        double* U = (double*)malloc(sizeof(double) * (size_t)C * dv);
        double* Wk = (double*)malloc(sizeof(double) * (size_t)C * dk);
        double* W = (double*)malloc(sizeof(double) * (size_t)C * dv);
        if (!S0 || !Snext || !Gam || !D || !A || !U || !Wk || !W) {
            free(S0); free(Snext); free(Gam); free(D); free(A); free(U); free(Wk); free(W);
#pragma omp atomic write
            failed = 1;
            continue;
        }
        if (init_state)
            memcpy(S0, init_state + ((size_t)n * H + h) * sz, sizeof(double) * sz);
        else
            memset(S0, 0, sizeof(double) * sz);

        int64_t t_begin = seq_start[n], t_end = seq_start[n + 1];
        int64_t ci = 0;
        for (int64_t t0 = t_begin; t0 < t_end; t0 += C, ++ci) {
            int L = (int)((t_end - t0) < C ? (t_end - t0) : C);
#define IDX_K(t) (((size_t)(t) * H + h) * dk)
#define IDX_V(t) (((size_t)(t) * H + h) * dv)
            if (s_chunk)
                memcpy(s_chunk + ((size_t)(chunk_base[n] + ci) * H + h) * sz, S0, sizeof(double) * sz);
            /* cumulative log decay (intermediate only) */
            if (g_out) {
                for (int c = 0; c < dk; ++c) {
                    double acc = 0.0;
                    for (int r = 0; r < L; ++r) {
                        acc += log_alpha[IDX_K(t0 + r) + c];
                        g_out[IDX_K(t0 + r) + c] = acc;
                    }
                }
            }
            /* Gam_r = prod_{j<=r} alpha_j */
            for (int c = 0; c < dk; ++c) {
                double acc = 1.0;
                for (int r = 0; r < L; ++r) {
                    acc *= exp(log_alpha[IDX_K(t0 + r) + c]);
                    Gam[(size_t)r * dk + c] = acc;
                }
            }
            /* D(r,i) = prod_{i<j<=r} alpha_j, built from D(r-1,i) */
            for (int i = 0; i < L; ++i) {
                for (int c = 0; c < dk; ++c) D[((size_t)i * C + i) * dk + c] = 1.0;
                for (int r = i + 1; r < L; ++r)
                    for (int c = 0; c < dk; ++c)
                        D[((size_t)r * C + i) * dk + c] =
                            D[((size_t)(r - 1) * C + i) * dk + c] * exp(log_alpha[IDX_K(t0 + r) + c]);
            }
            /* A[r,i], strictly lower */
            for (int r = 0; r < L; ++r) {
                double br = beta[(size_t)(t0 + r) * H + h];
                for (int i = 0; i < L; ++i) {
                    double s = 0.0;
                    if (i < r)
                        for (int c = 0; c < dk; ++c)
                            s += k[IDX_K(t0 + r) + c] * k[IDX_K(t0 + i) + c] * D[((size_t)r * C + i) * dk + c];
                    A[(size_t)r * C + i] = br * s;
                }
            }
            /* forward substitution: (I + A) U = Diag(beta) V, (I + A) Wk = Diag(beta)(K . Gam) */
            for (int r = 0; r < L; ++r) {
                double br = beta[(size_t)(t0 + r) * H + h];
                for (int j = 0; j < dv; ++j) {
                    double s = br * v[IDX_V(t0 + r) + j];
                    for (int i = 0; i < r; ++i) s -= A[(size_t)r * C + i] * U[(size_t)i * dv + j];
                    U[(size_t)r * dv + j] = s;
                }
                for (int c = 0; c < dk; ++c) {
                    double s = br * k[IDX_K(t0 + r) + c] * Gam[(size_t)r * dk + c];
                    for (int i = 0; i < r; ++i) s -= A[(size_t)r * C + i] * Wk[(size_t)i * dk + c];
                    Wk[(size_t)r * dk + c] = s;
                }
            }
            /* W = U - Wk S0 */
            for (int r = 0; r < L; ++r)
                for (int j = 0; j < dv; ++j) {
                    double s = U[(size_t)r * dv + j];
                    for (int c = 0; c < dk; ++c) s -= Wk[(size_t)r * dk + c] * S0[(size_t)c * dv + j];
                    W[(size_t)r * dv + j] = s;
                }
            /* outputs: inter-chunk term plus masked intra-chunk term (i <= r) */
            for (int r = 0; r < L; ++r) {
                double* orow = o + IDX_V(t0 + r);
                for (int j = 0; j < dv; ++j) {
                    double s = 0.0;
                    for (int c = 0; c < dk; ++c)
                        s += q[IDX_K(t0 + r) + c] * Gam[(size_t)r * dk + c] * S0[(size_t)c * dv + j];
                    orow[j] = s;
                }
                for (int i = 0; i <= r; ++i) {
                    double p_ri = 0.0;
                    for (int c = 0; c < dk; ++c)
                        p_ri += q[IDX_K(t0 + r) + c] * k[IDX_K(t0 + i) + c] * D[((size_t)r * C + i) * dk + c];
                    for (int j = 0; j < dv; ++j) orow[j] += p_ri * W[(size_t)i * dv + j];
                }
            }
            /* next chunk start state */
            for (int c = 0; c < dk; ++c)
                for (int j = 0; j < dv; ++j) {
                    double s = Gam[(size_t)(L - 1) * dk + c] * S0[(size_t)c * dv + j];
                    for (int i = 0; i < L; ++i)
                        s += k[IDX_K(t0 + i) + c] * D[((size_t)(L - 1) * C + i) * dk + c] * W[(size_t)i * dv + j];
                    Snext[(size_t)c * dv + j] = s;
                }
            if (u_out)
                for (int r = 0; r < L; ++r) memcpy(u_out + IDX_V(t0 + r), U + (size_t)r * dv, sizeof(double) * dv);
            if (wk_out)
                for (int r = 0; r < L; ++r) memcpy(wk_out + IDX_K(t0 + r), Wk + (size_t)r * dk, sizeof(double) * dk);
            if (w_out)
                for (int r = 0; r < L; ++r) memcpy(w_out + IDX_V(t0 + r), W + (size_t)r * dv, sizeof(double) * dv);
            memcpy(S0, Snext, sizeof(double) * sz);
#undef IDX_K
#undef IDX_V
        }
        if (final_state) memcpy(final_state + ((size_t)n * H + h) * sz, S0, sizeof(double) * sz);
        free(S0); free(Snext); free(Gam); free(D); free(A); free(U); free(Wk); free(W);
    }
    free(chunk_base);
    return failed ? -2 : 0;
}

/* ------------------------------------------------------------------------
 * O3: reverse-mode gradient of O1 (the token recurrence), for training.
 *
 * The pages say training needs the chunkwise parallel form but derive no
 * backward pass; this is the chain rule applied to O1's steps, in reverse
 * token order.  For token t, with S_prev the state before it and G the
 * gradient with respect to the state after it:
 *   dq_t   = S_t do_t                    (o_t = S_t^T q_t)
 *   G     += q_t do_t^T
 *   Sd     = Diag(alpha_t) S_prev,  u = v_t - Sd^T k_t
 *   dbeta_t = k_t^T G u
 *   du     = beta_t G^T k_t,  dv_t = du
 *   dk_t   = beta_t G u - Sd du
 *   dSd    = G - k_t du^T
 *   dlog_alpha_t[c] = sum_j dSd[c][j] Sd[c][j]
 *   G      = Diag(alpha_t) dSd           (gradient with respect to S_prev)
 * and d init_state = G after the first token.  The loss is
 *   L = sum(do * o) + sum(d_final_state * final_state).
 * States are recomputed forward from a copy kept every 64 tokens (the same
 * values as one forward pass; the copies only bound the memory).
 * ------------------------------------------------------------------------ */
int kda_ref_backward_f64(const double* q, const double* k, const double* v,
                         const double* log_alpha, const double* beta,
                         const double* init_state, const int64_t* seq_start,
                         int n_seqs, int H, int dk, int dv,
                         const double* d_o, const double* d_final_state,
                         double* dq, double* dkk, double* dvv, double* dla, double* dbeta,
                         double* d_init_state, int n_threads)
{
    enum { KB = 64 };
    if (n_seqs < 0 || H <= 0 || dk <= 0 || dv <= 0) return -1;
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#else
    (void)n_threads;
#endif
    const size_t sz = (size_t)dk * dv;
    long n_pairs = (long)n_seqs * H;
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (long p = 0; p < n_pairs; ++p) {
        int n = (int)(p / H), h = (int)(p % H);
        int64_t t_begin = seq_start[n], t_end = seq_start[n + 1], len = t_end - t_begin;
        int64_t n_blk = (len + KB - 1) / KB;
        double* ckpt = (double*)malloc(sizeof(double) * sz * (size_t)(n_blk > 0 ? n_blk : 1));
        double* st = (double*)malloc(sizeof(double) * sz * (KB + 1));   /* states of one block */
        double* G = (double*)malloc(sizeof(double) * sz);
        double* dSd = (double*)malloc(sizeof(double) * sz);
        double* a = (double*)malloc(sizeof(double) * (size_t)dk);
        double* r = (double*)malloc(sizeof(double) * (size_t)(dv > dk ? dv : dk));
        double* u = (double*)malloc(sizeof(double) * (size_t)dv);
        double* du = (double*)malloc(sizeof(double) * (size_t)dv);
        double* Gu = (double*)malloc(sizeof(double) * (size_t)dk);
        if (!ckpt || !st || !G || !dSd || !a || !r || !u || !du || !Gu) {
            free(ckpt); free(st); free(G); free(dSd); free(a); free(r); free(u); free(du); free(Gu);
#pragma omp atomic write
            failed = 1;
            continue;
        }
        /* one step of O1: S (in place) from the state before token t */
#define STEP(S, t)                                                                          \
        do {                                                                                \
            const double* kt_ = k + ((size_t)(t) * H + h) * dk;                             \
            const double* vt_ = v + ((size_t)(t) * H + h) * dv;                             \
            const double* lat_ = log_alpha + ((size_t)(t) * H + h) * dk;                    \
            double bt_ = beta[(size_t)(t) * H + h];                                         \
            for (int c = 0; c < dk; ++c) a[c] = exp(lat_[c]);                               \
            for (int c = 0; c < dk; ++c)                                                    \
                for (int j = 0; j < dv; ++j) (S)[(size_t)c * dv + j] *= a[c];               \
            for (int j = 0; j < dv; ++j) r[j] = 0.0;                                        \
            for (int c = 0; c < dk; ++c)                                                    \
                for (int j = 0; j < dv; ++j) r[j] += (S)[(size_t)c * dv + j] * kt_[c];      \
            for (int c = 0; c < dk; ++c)                                                    \
                for (int j = 0; j < dv; ++j) (S)[(size_t)c * dv + j] += bt_ * kt_[c] * (vt_[j] - r[j]); \
        } while (0)

        /* forward: the state at the start of every block of KB tokens */
        if (init_state) memcpy(st, init_state + ((size_t)n * H + h) * sz, sizeof(double) * sz);
        else memset(st, 0, sizeof(double) * sz);
        for (int64_t b = 0; b < n_blk; ++b) {
            memcpy(ckpt + (size_t)b * sz, st, sizeof(double) * sz);
            int64_t t0 = t_begin + b * KB, t1 = t0 + KB < t_end ? t0 + KB : t_end;
            for (int64_t t = t0; t < t1; ++t) STEP(st, t);
        }
        /* G = gradient with respect to the final state */
        if (d_final_state) memcpy(G, d_final_state + ((size_t)n * H + h) * sz, sizeof(double) * sz);
        else memset(G, 0, sizeof(double) * sz);
        for (int64_t b = n_blk - 1; b >= 0; --b) {
            int64_t t0 = t_begin + b * KB, t1 = t0 + KB < t_end ? t0 + KB : t_end;
            /* st[i] = state after i tokens of the block */
            memcpy(st, ckpt + (size_t)b * sz, sizeof(double) * sz);
            for (int64_t t = t0; t < t1; ++t) {
                double* nx = st + (size_t)(t - t0 + 1) * sz;
                memcpy(nx, nx - sz, sizeof(double) * sz);
                STEP(nx, t);
            }
            for (int64_t t = t1 - 1; t >= t0; --t) {
                const double* Sprev = st + (size_t)(t - t0) * sz;
                const double* St = Sprev + sz;
                const double* qt = q + ((size_t)t * H + h) * dk;
                const double* kt = k + ((size_t)t * H + h) * dk;
                const double* vt = v + ((size_t)t * H + h) * dv;
                const double* lat = log_alpha + ((size_t)t * H + h) * dk;
                const double* dot = d_o + ((size_t)t * H + h) * dv;
                double bt = beta[(size_t)t * H + h];
                double* dqt = dq + ((size_t)t * H + h) * dk;
                double* dkt = dkk + ((size_t)t * H + h) * dk;
                double* dvt = dvv + ((size_t)t * H + h) * dv;
                double* dlat = dla + ((size_t)t * H + h) * dk;
                /* output: dq_t = S_t do_t, G += q_t do_t^T */
                for (int c = 0; c < dk; ++c) {
                    double acc = 0.0;
                    for (int j = 0; j < dv; ++j) acc += St[(size_t)c * dv + j] * dot[j];
                    dqt[c] = acc;
                }
                for (int c = 0; c < dk; ++c)
                    for (int j = 0; j < dv; ++j) G[(size_t)c * dv + j] += qt[c] * dot[j];
                /* Sd = Diag(alpha) S_prev (kept in dSd for now), u = v - Sd^T k */
                for (int c = 0; c < dk; ++c) a[c] = exp(lat[c]);
                for (int c = 0; c < dk; ++c)
                    for (int j = 0; j < dv; ++j) dSd[(size_t)c * dv + j] = a[c] * Sprev[(size_t)c * dv + j];
                for (int j = 0; j < dv; ++j) {
                    double acc = 0.0;
                    for (int c = 0; c < dk; ++c) acc += dSd[(size_t)c * dv + j] * kt[c];
                    u[j] = vt[j] - acc;
                }
                /* Gu = G u, r = G^T k */
                for (int c = 0; c < dk; ++c) {
                    double acc = 0.0;
                    for (int j = 0; j < dv; ++j) acc += G[(size_t)c * dv + j] * u[j];
                    Gu[c] = acc;
                }
                for (int j = 0; j < dv; ++j) {
                    double acc = 0.0;
                    for (int c = 0; c < dk; ++c) acc += G[(size_t)c * dv + j] * kt[c];
                    r[j] = acc;
                }
                double db = 0.0;
                for (int c = 0; c < dk; ++c) db += kt[c] * Gu[c];
                dbeta[(size_t)t * H + h] = db;
                for (int j = 0; j < dv; ++j) { du[j] = bt * r[j]; dvt[j] = du[j]; }
                for (int c = 0; c < dk; ++c) {
                    double acc = 0.0;
                    for (int j = 0; j < dv; ++j) acc += dSd[(size_t)c * dv + j] * du[j];
                    dkt[c] = bt * Gu[c] - acc;
                }
                /* dSd = G - k du^T; dlog_alpha = rowsum(dSd . Sd); G = Diag(alpha) dSd */
                for (int c = 0; c < dk; ++c) {
                    double acc = 0.0;
                    for (int j = 0; j < dv; ++j) {
                        double sd = dSd[(size_t)c * dv + j];
                        double g = G[(size_t)c * dv + j] - kt[c] * du[j];
                        acc += g * sd;
                        G[(size_t)c * dv + j] = a[c] * g;
                    }
                    dlat[c] = acc;
                }
            }
        }
#undef STEP
        if (d_init_state) memcpy(d_init_state + ((size_t)n * H + h) * sz, G, sizeof(double) * sz);
        free(ckpt); free(st); free(G); free(dSd); free(a); free(r); free(u); free(du); free(Gu);
    }
    return failed ? -2 : 0;
}

/* Number of threads the OpenMP runtime would use (1 without OpenMP). */
int kda_ref_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
