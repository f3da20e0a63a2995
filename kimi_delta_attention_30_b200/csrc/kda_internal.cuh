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

    __device__ __forceinline__ void locate(int chunk, int& seq, int& tok0, int& len, int& idx) const {
        if (seqs == nullptr) {
            seq = chunk / ncps;
            idx = chunk - seq * ncps;
            tok0 = seq * T + idx * C;
            len = min(C, T - idx * C);
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

// ---- optional per-kernel timing hook (see kda_set_timing_events) -----------

struct TimingHook {
    void* ev[32];
    int n;
};
TimingHook& timing_hook();   // per host thread

// Record hook event i on `s` if the hook asks for it.
inline void timing_mark(cudaStream_t s, int i) {
    TimingHook& h = timing_hook();
    if (i < h.n && h.ev[i]) cudaEventRecord((cudaEvent_t)h.ev[i], s);
}

// ---- launchers (return cudaSuccess or the launch error) --------------------

struct SimtWorkspace {
    float* g;
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

cudaError_t launch_decode(kda_dtype dtype, const void* q, const void* k, const void* v,
                          const void* log_alpha, const void* beta, float* state, int N, int H,
                          int dk, int dv, void* o, cudaStream_t stream);

}  // namespace kda
