// Internal declarations shared by the KDA CUDA sources (not part of the ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kda.h"

namespace kda {

// One sequence of a batch: token offset, length, index of its first chunk in
// the global chunk numbering, and its index in the caller's batch.
struct SeqInfo {
    int tok0;
    int len;
    int chunk0;
    int seq;
};

// Maps a global chunk index to its sequence and token range.  Equal-length
// batches (seqs == nullptr) use arithmetic; packed batches search `seqs`
// (natural order, chunk0 non-decreasing).
struct ChunkMap {
    const SeqInfo* seqs;
    int n_seqs;
    int T;          // tokens per sequence (equal-length case)
    int C;
    int ncps;       // chunks per sequence (equal-length case)
    // packed batches: per chunk (first token, length, sequence, index in the sequence),
    // filled once per call so that a kernel's first loads wait on one lookup instead of
    // a search's chain of dependent loads; nullptr falls back to the search
    const int4* chunks = nullptr;

    __device__ __forceinline__ void locate(int chunk, int& seq, int& tok0, int& len, int& idx) const {
        if (seqs == nullptr) {
            seq = chunk / ncps;
            idx = chunk - seq * ncps;
            tok0 = seq * T + idx * C;
            len = min(C, T - idx * C);
        } else if (chunks != nullptr) {
            const int4 e = __ldg(chunks + chunk);
            tok0 = e.x;
            len = e.y;
            seq = e.z;
            idx = e.w;
        } else {
            int lo = 0, hi = n_seqs - 1;
            while (lo < hi) {            // last s with chunk0 <= chunk
                int mid = (lo + hi + 1) >> 1;
                if (__ldg(&seqs[mid].chunk0) <= chunk) lo = mid; else hi = mid - 1;
            }
            SeqInfo s = seqs[lo];
            seq = s.seq;
            idx = chunk - s.chunk0;
            tok0 = s.tok0 + idx * C;
            len = min(C, s.len - idx * C);
        }
    }
};

// Sequence descriptor for kernels that walk one sequence (state carry):
// `order` lists sequences longest first; nullptr means equal-length batch.
struct SeqMap {
    const SeqInfo* order;
    int T;
    int C;
    int ncps;

    __device__ __forceinline__ SeqInfo get(int rank) const {
        if (order == nullptr) {
            SeqInfo s;
            s.tok0 = rank * T;
            s.len = T;
            s.chunk0 = rank * ncps;
            s.seq = rank;
            return s;
        }
        return order[rank];
    }
};

template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// log(alpha) floor used by every kernel: exp(-100) ~ 3.7e-44 is below the
// smallest fp32 normal number, so the clamp is invisible in fp32 results while
// keeping cumulative sums finite when alpha = 0 (log alpha = -inf).
constexpr float kLogAlphaFloor = -100.0f;

// 2^x on the special-function unit (PTX ex2.approx: about 22 correct bits;
// subnormal results flush to 0).
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
constexpr float kLog2e = 1.4426950408889634f;

// ---- fused input preprocessing (kda_prep flags) --------------------------------
// log(1 + u) for u in [0, 1] as u q(u): q of degree 8 is the Chebyshev interpolant
// of log(1 + u) / u at 400 Chebyshev nodes of [0, 1], rewritten in powers of u.
// In fp32 with fused multiply-adds the absolute error is at most 1.2e-7 (relative
// 2e-7, and relative 1e-7 as u -> 0), checked in fp64 at 2e6 points.  It runs on
// the FMA pipe, leaving the special-function unit one 2^x per gate value.
__host__ __device__ constexpr float l1p_coef(int i) {
    return i == 0 ? 1.000000000e+00f : i == 1 ? -4.999950230e-01f : i == 2 ? 3.331927061e-01f
         : i == 3 ? -2.484436929e-01f : i == 4 ? 1.911143064e-01f : i == 5 ? -1.367477030e-01f
         : i == 6 ? 7.836166769e-02f : i == 7 ? -2.958850749e-02f : 5.253457930e-03f;
}
__device__ __forceinline__ float log1p_unit(float u) {
    float p = l1p_coef(8);
#pragma unroll
    for (int i = 7; i >= 0; --i) p = fmaf(p, u, l1p_coef(i));
    return p * u;
}
// -softplus(a) = -log(1 + e^a), split as max(a, 0) + log(1 + e^-|a|) so that
// nothing overflows (e^-|a| in (0, 1]).
__device__ __forceinline__ float neg_softplus(float a) {
    return -(fmaxf(a, 0.f) + log1p_unit(ex2_approx(-fabsf(a) * kLog2e)));
}
// log alpha from the log_alpha argument: as given, or -softplus of a raw gate
// logit; then the floor every kernel applies.
__device__ __forceinline__ float prep_log_alpha(float x, unsigned prep) {
    if (prep & KDA_PREP_GATE_SOFTPLUS) x = neg_softplus(x);
    return fmaxf(x, kLogAlphaFloor);
}
// beta from the beta argument: as given, or the logistic function of a raw logit.
__device__ __forceinline__ float prep_beta(float x, unsigned prep) {
    return (prep & KDA_PREP_BETA_SIGMOID) ? 1.f / (1.f + expf(-x)) : x;
}
// 1 / ||x|| for the key/query normalisation (0 for an all-zero vector).
__device__ __forceinline__ float inv_norm_from_sq(float sum_sq) { return sum_sq > 0.f ? rsqrtf(sum_sq) : 0.f; }

// ---- cumulative decays as fp32 (hi, lo) pairs -------------------------------
// Within a chunk g reaches -100 and beyond, where one fp32 ulp is ~1e-5; a decay
// exp(g_a - g_b) formed from two rounded g would carry that as a relative error.
// The CUDA-core kernels therefore keep g as hi + lo (the fp64 cumulative sum split
// in two floats) and form differences as (hi_a - hi_b) + (lo_a - lo_b).
// Both use 2^x on the SFU: a relative error near 2^-22, plus the rounding of the
// exponent times log2 e (3e-7 relative at |exponent| = 5, where terms still count).
__device__ __forceinline__ float exp_gdiff(float ah, float al, float bh, float bl) {
    return ex2_approx(((ah - bh) + (al - bl)) * kLog2e);
}
// exp(g) for g = hi + lo, |lo| <= ulp(hi) / 2: exp(hi) (1 + lo) to second order.
__device__ __forceinline__ float exp_g(float h, float l) { return ex2_approx(h * kLog2e) * (1.f + l); }

// ---- optional per-kernel timing hook (see kda_set_timing_events) -----------

struct TimingHook {
    void* ev[32];
    int n;
    int base;   // kernels launched by the call before the algorithm's own (sequence tables)
};
TimingHook& timing_hook();   // per host thread

// Record hook event `i` (counted from the call's first launch) on `s` if the hook asks for it.
inline void timing_mark_abs(cudaStream_t s, int i) {
    TimingHook& h = timing_hook();
    if (i >= 0 && i < h.n && i < 32 && h.ev[i]) cudaEventRecord((cudaEvent_t)h.ev[i], s);
}
// The same for the algorithm's own kernels: mark i follows its i-th kernel.
inline void timing_mark(cudaStream_t s, int i) { timing_mark_abs(s, i == 0 ? 0 : timing_hook().base + i); }

// ---- launchers (return cudaSuccess or the launch error) --------------------

struct SimtWorkspace {
    float* g;        // cumulative log decay, high part (fp32 rounding of the fp64 sum)
    float* gl;       // low part: g = g + gl to about 48 bits
    float* U;
    float* Wk;
    float* W;
    float* S_chunk;
};

cudaError_t launch_simt_prefill(kda_dtype dtype, const void* q, const void* k, const void* v,
                                const void* log_alpha, const void* beta, const float* init_state,
                                void* o, float* final_state, const ChunkMap& cmap, const SeqMap& smap,
                                int n_chunks, int n_seqs, int H, int dk, int dv, int C,
                                const SimtWorkspace& ws, cudaStream_t stream);

// The CUDA-core forward without the output kernel: g, U, Wk, W and every
// chunk's start state into `ws` (for the backward pass).
cudaError_t launch_simt_states(kda_dtype dtype, const void* k, const void* v, const void* log_alpha,
                               const void* beta, const float* init_state, const ChunkMap& cmap, const SeqMap& smap,
                               int n_chunks, int n_seqs, int H, int dk, int dv, int C, const SimtWorkspace& ws,
                               cudaStream_t stream);

// Backward scratch (fp32): the forward intermediates plus the gradients the
// backward kernels hand to one another.
struct BwdWorkspace {
    SimtWorkspace fwd;  // g, U, Wk, W [tokens, H, d]; S_chunk [chunks, H, dk, dv]
    float* dS_chunk;    // [chunks, H, dk, dv] gradient w.r.t. each chunk's end state
    float* dW;          // [tokens, H, dv]
    float* P;           // [chunks, H, C, C] decayed causal scores
    float* dQg;         // [tokens, H, dk]
    float* dKd;         // [tokens, H, dk]
    float* dWk;         // [tokens, H, dk]
    float* dKg;         // [tokens, H, dk]
    float* dGam;        // [chunks, H, dk]
    float* dAt;         // [chunks, H, C, C] gradient w.r.t. the unscaled key products
    float* At;          // [chunks, H, C, C] the unscaled key products (strictly lower)
    float* Qg;          // [tokens, H, dk] q . exp(g)
    float* Kd;          // [tokens, H, dk] k . exp(g_C - g)
    void* tc_ws;        // tensor-core workspace for the recompute (bf16, d = 128), or null
    float* T;           // [chunks, H, C, C] (I + A)^-1 from that recompute (tensor-core path only)
    void* o_scratch;    // outputs of that recompute [tokens, H, dv] bf16 (unused)
};

// g only (the CUDA-core K1), into ws.g / ws.gl.
cudaError_t launch_simt_g(kda_dtype dtype, const void* log_alpha, const ChunkMap& cmap, int n_chunks, int H, int dk,
                          const SimtWorkspace& ws, cudaStream_t stream);

// Tensor-core recompute for the backward pass (bf16, d = 128): the per-chunk
// images in tc_ws, T and the key products, and the chunk start states and W
// from the state carry.
cudaError_t launch_tc_states(const void* q, const void* k, const void* v, const void* log_alpha, const void* beta,
                             const float* init_state, void* o_scratch, const ChunkMap& cmap, const SeqMap& smap,
                             int n_chunks, int n_seqs, int H, void* tc_ws, float* S_chunk, float* W,
                             float* T_store, float* At_store, cudaStream_t stream);

cudaError_t launch_simt_backward(kda_dtype dtype, const void* q, const void* k, const void* v,
                                 const void* log_alpha, const void* beta, const float* init_state,
                                 const void* d_o, const float* d_final_state, void* dq, void* dk, void* dv,
                                 void* dlog_alpha, void* dbeta, float* d_init_state, const ChunkMap& cmap,
                                 const SeqMap& smap, int n_chunks, int n_seqs, int H, int dkk, int dvv, int C,
                                 const BwdWorkspace& ws, cudaStream_t stream);

// Tensor-core chunk-local products of the backward pass (bf16, d = 128):
// dQg = dO S^T, dWk = -dW S^T, dKd = W dS'^T, dP = dO W^T, dGam = rowsum(dS' . S).
// Tensor-core reverse chain of the backward pass (bf16, d = 128): from the
// per-chunk images of the recompute, dW = Kd dS' + P^T dO and dS = Gamma dS' +
// Qg^T dO - Wk^T dW per chunk, storing dS_chunk, dW and the initial-state gradient.
cudaError_t launch_tc_chain(void* tc_ws, const void* d_o, const float* d_final, float* dS_chunk, float* dW,
                            float* d_init, const SeqMap& smap, int n_seqs, int H, cudaStream_t stream);

// Tensor-core back substitution of the backward pass (bf16, d = 128):
// [Y | Z] = T^T [dW | dWk], dA = -(Y U^T + Z Wk^T) (i < r), dv = beta Y, dKg = beta Z,
// dbeta_r = v_r.Y_r + Kg_r.Z_r + sum_i dA_ri At_ri, dAt = Diag(beta) dA.
cudaError_t launch_kb_b_tc(const float* T, const float* At, const void* tc_ws, const float* dW,
                           const float* dWk, const void* k, const void* v, const void* beta, const float* g,
                           const float* gl, void* dv_out, void* dbeta_out, float* dKg, float* dAt, int* err,
                           const ChunkMap& cmap, int n_chunks, int H, cudaStream_t stream);

cudaError_t launch_kb_a_tc(const void* d_o, const float* W, const float* dW, const float* S_chunk,
                           const float* dS_chunk, float* dQg, float* dKd, float* dWk, float* dGam, float* dP, int* err,
                           const ChunkMap& cmap, int n_chunks, int H, cudaStream_t stream);

// Tensor-core pairwise gradient terms of the backward pass (bf16, d = 128): from dAt,
// dP (strictly lower parts in the products, dP's diagonal elementwise) and the
// gradients of the elementwise factors, dq, dk and dlog alpha.
cudaError_t launch_kb_c_tc(const void* q, const void* k, const void* la, const float* g, const float* gl,
                           const float* dAt, const float* dP, const float* dQg, const float* dKd, const float* dKg,
                           const float* dGam, void* dq, void* dk, void* dla, int* err, const ChunkMap& cmap,
                           int n_chunks, int H, cudaStream_t stream);

// A segment's affine map S_end = M S_start + F (M [N, H, dk, dk], F [N, H, dk, dv]).
cudaError_t launch_tc_segment_map(const void* q, const void* k, const void* v, const void* log_alpha,
                                  const void* beta, const ChunkMap& cmap, const SeqMap& smap, int n_chunks,
                                  int n_seqs, int H, void* tc_ws, float* M, float* F, cudaStream_t stream);
cudaError_t launch_simt_segment_map(kda_dtype dtype, const void* k, const void* v, const void* log_alpha,
                                    const void* beta, const ChunkMap& cmap, const SeqMap& smap, int n_chunks,
                                    int n_seqs, int H, int dk, int dv, int C, const SimtWorkspace& ws, float* Mmap,
                                    float* F, cudaStream_t stream);
// states[0] = init (or 0), states[r + 1] = M_r states[r] + F_r, r < R.
cudaError_t launch_compose_states(const float* M, const float* F, const float* init, int R, int N, int H, int dk,
                                  int dv, float* out, cudaStream_t stream);

cudaError_t launch_decode(kda_dtype dtype, const void* q, const void* k, const void* v,
                          const void* log_alpha, const void* beta, float* state, int N, int H,
                          int dk, int dv, void* o, unsigned prep, cudaStream_t stream);

}  // namespace kda
