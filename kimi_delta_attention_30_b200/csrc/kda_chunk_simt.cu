// CUDA-core (SIMT, fp32 arithmetic) chunkwise KDA prefill: four kernels that
// exchange their intermediates through the workspace.
//
//   K1 cumulative log decay  g_r = sum_{j<=r} log alpha_j   (restarting per chunk)
//   K2 WY/UT transform       A_{r,i} = beta_r sum_c k_rc k_ic exp(g_rc - g_ic), i < r
//                            (I + A) U  = Diag(beta) V
//                            (I + A) Wk = Diag(beta) (K . exp(g))
//   K3 state carry           for each chunk in order: S_n -> workspace,
//                            W = U - Wk S_n,
//                            S_{n+1} = Diag(exp(g_C)) S_n + (K . exp(g_C - g))^T W
//   K4 output                O = (Q . exp(g)) S_n + (M_incl . [(Q x K) exp(g_r - g_i)]) W
//
// Chunkwise form: "From GPT-2 to Kimi K3" essay (pwwt.cn/news/3716252),
// chunkwise and Gated DeltaNet paragraphs (masked attention inside a chunk,
// state-first recurrence across chunks, cumulative decay factors across
// chunks); WY / DPLR restructuring: "我终于看懂了 KDA" explainer
// (pwwt.cn/news/3787313), sections 16-17.  This path evaluates every decay
// as exp of a non-positive difference g_r - g_i (r >= i), so it is exact for
// any decay range, with g summed in fp64 and kept as an fp32 (hi, lo) pair so
// that the difference keeps its accuracy when g itself is large; it serves the
// fp32 inputs and is the CUDA-core reference for the tensor-core path.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kThreadsW = 512;   // threads per block: the kernels' loops are latency bound
constexpr int kBV = 32;   // d_v columns per state-carry block
constexpr int kMaxDK = 128;

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// K1: one block per (chunk, head), one thread per key channel.
template <typename Tin>
__global__ void __launch_bounds__(128) k1_cumsum(const Tin* __restrict__ la, float* __restrict__ g,
                                                 float* __restrict__ gl, ChunkMap cmap, int H, int dk) {
    int seq, tok0, len, idx;
    cmap.locate(blockIdx.x, seq, tok0, len, idx);
    const int h = blockIdx.y, c = threadIdx.x;
    double acc = 0.0;
    for (int r = 0; r < len; ++r) {
        size_t off = ((size_t)(tok0 + r) * H + h) * dk + c;
        acc += (double)fmaxf(to_f32(la[off]), kLogAlphaFloor);
        const float hi = (float)acc;
        g[off] = hi;
        gl[off] = (float)(acc - (double)hi);
    }
}

// K2: one block per (chunk, head).  Dynamic shared memory:
//   A [C][C] | phase 1: Ks, Gs [C][dk], GLs [C][dk] (bf16)  / phase 2: X [C][dk + dv]
// (the low part of g is staged in bf16: |lo| <= ulp(g) / 2, so bf16 keeps it to
// ulp(g) 2^-10, below 3e-8 for |g| < 256, and 128-token chunks fit at d = 128)
template <typename Tin>
__global__ void __launch_bounds__(kThreadsW) k2_wy(const Tin* __restrict__ k, const Tin* __restrict__ v,
                                                  const Tin* __restrict__ beta, const float* __restrict__ g,
                                                  const float* __restrict__ gl, float* __restrict__ U,
                                                  float* __restrict__ Wk, ChunkMap cmap, int H, int dk, int dv,
                                                  int C) {
    extern __shared__ float smem[];
    int seq, tok0, len, idx;
    cmap.locate(blockIdx.x, seq, tok0, len, idx);
    const int h = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    float* A = smem;
    float* Ks = A + C * C;
    float* Gs = Ks + C * dk;
    __nv_bfloat16* GLs = reinterpret_cast<__nv_bfloat16*>(Gs + C * dk);

    for (int e = tid; e < len * dk; e += kThreadsW) {
        int r = e / dk, c = e - r * dk;
        size_t off = ((size_t)(tok0 + r) * H + h) * dk + c;
        Ks[r * dk + c] = to_f32(k[off]);
        Gs[r * dk + c] = g[off];
        GLs[r * dk + c] = __float2bfloat16_rn(gl[off]);
    }
    __syncthreads();
    // A, one warp per (r, i) pair, lanes over channels
    for (int p = warp; p < len * len; p += kThreadsW / 32) {
        int r = p / len, i = p - r * len;
        float s = 0.f;
        if (i < r) {
            for (int c = lane; c < dk; c += 32)
                s += Ks[r * dk + c] * Ks[i * dk + c] *
                     exp_gdiff(Gs[r * dk + c], __bfloat162float(GLs[r * dk + c]), Gs[i * dk + c],
                               __bfloat162float(GLs[i * dk + c]));
            s = warp_sum(s) * to_f32(beta[(size_t)(tok0 + r) * H + h]);
        }
        if (lane == 0) A[r * C + i] = s;
    }
    __syncthreads();
    // forward substitution: the right-hand sides [beta V | beta K exp(g)] are loaded
    // whole (X reuses the Ks/Gs region), then one column per thread, in place
    float* X = Ks;
    const int ncol = dk + dv;
    for (int e = tid; e < len * ncol; e += kThreadsW) {
        const int r = e / ncol, j = e - r * ncol;
        const size_t tok = (size_t)(tok0 + r) * H + h;
        const float br = to_f32(beta[tok]);
        if (j < dv) {
            X[e] = br * to_f32(v[tok * dv + j]);
        } else {
            const int c = j - dv;
            X[e] = br * to_f32(k[tok * dk + c]) * exp_g(g[tok * dk + c], gl[tok * dk + c]);
        }
    }
    __syncthreads();
    for (int j = tid; j < ncol; j += kThreadsW) {
        for (int r = 1; r < len; ++r) {
            float s = X[r * ncol + j];
            for (int i = 0; i < r; ++i) s -= A[r * C + i] * X[i * ncol + j];
            X[r * ncol + j] = s;
        }
    }
    __syncthreads();
    for (int e = tid; e < len * ncol; e += kThreadsW) {
        const int r = e / ncol, j = e - r * ncol;
        const size_t tok = (size_t)(tok0 + r) * H + h;
        if (j < dv) U[tok * dv + j] = X[e];
        else Wk[tok * dk + (j - dv)] = X[e];
    }
}

// K3: one block per (sequence, head, d_v tile of kBV columns), sequential over
// the sequence's chunks.  Shared: S [dk][kBV], M [C][dk] (Wk, then K . decay),
// Ws [C][kBV], gC, gCl [dk].
// MAP (a segment's affine map S_end = Mmap S_start + F): blockIdx.z < dv / kBV
// carries the state from zero (F, into final_state [N, H, dk, dv]); the next
// dk / kBV tiles carry the columns of the identity without the values' term U
// (Mmap, into map_out [N, H, dk, dk]); nothing else is stored.
template <typename Tin, int CC, bool MAP = false>
__global__ void __launch_bounds__(kThreadsW, 2) k3_state(const Tin* __restrict__ k, const float* __restrict__ g,
                                                     const float* __restrict__ gl,
                                                     const float* __restrict__ U, const float* __restrict__ Wkg,
                                                     float* __restrict__ Wg, float* __restrict__ S_chunk,
                                                     const float* __restrict__ init_state,
                                                     float* __restrict__ final_state, SeqMap smap, int H, int dk,
                                                     int dv, int C, float* __restrict__ map_out) {
    extern __shared__ float smem[];
    const SeqInfo sq = smap.get(blockIdx.x);
    const bool mcols = MAP && (int)blockIdx.z >= dv / kBV;
    const int h = blockIdx.y, j0 = (mcols ? (int)blockIdx.z - dv / kBV : (int)blockIdx.z) * kBV, tid = threadIdx.x;
    const int ld = mcols ? dk : dv;     // row length of this tile's state (F and S: dv; Mmap: dk)
    float* S = smem;
    float* M = S + dk * kBV;
    float* Ws = M + C * dk;
    float* gC = Ws + C * kBV;
    float* gCl = gC + dk;

    const size_t st_base = ((size_t)sq.seq * H + h) * dk * ld;
    for (int e = tid; e < dk * kBV; e += kThreadsW) {
        int c = e / kBV, j = e - c * kBV;
        if (MAP)
            S[e] = (mcols && c == j0 + j) ? 1.f : 0.f;
        else
            S[e] = init_state ? init_state[st_base + (size_t)c * dv + j0 + j] : 0.f;
    }
    __syncthreads();
    const int nch = (sq.len + C - 1) / C;
    for (int n = 0; n < nch; ++n) {
        const int t0 = sq.tok0 + n * C;
        const int L = min(C, sq.len - n * C);
        const size_t sc_base = ((size_t)(sq.chunk0 + n) * H + h) * dk * dv;
        if (!MAP) {
            for (int e = tid; e < dk * kBV; e += kThreadsW) {
                int c = e / kBV, j = e - c * kBV;
                S_chunk[sc_base + (size_t)c * dv + j0 + j] = S[e];
            }
        }
        for (int e = tid; e < L * dk; e += kThreadsW) {
            int r = e / dk, c = e - r * dk;
            M[e] = Wkg[((size_t)(t0 + r) * H + h) * dk + c];
        }
        __syncthreads();
        // W = U - Wk S: thread t forms column t % 32 of rows t / 32 + 16 m
        {
            const int j = tid & 31, r0 = tid >> 5;
            float acc[CC / 16];
#pragma unroll
            for (int m = 0; m < CC / 16; ++m) {
                const int r = r0 + 16 * m;
                acc[m] = (r < L && !mcols) ? U[((size_t)(t0 + r) * H + h) * dv + j0 + j] : 0.f;
            }
            for (int c = 0; c < dk; ++c) {
                const float sv = S[c * kBV + j];
#pragma unroll
                for (int m = 0; m < CC / 16; ++m) acc[m] -= M[(r0 + 16 * m) * dk + c] * sv;   // rows >= L unused
            }
#pragma unroll
            for (int m = 0; m < CC / 16; ++m) {
                const int r = r0 + 16 * m;
                if (r < L) {
                    Ws[r * kBV + j] = acc[m];
                    if (!MAP) Wg[((size_t)(t0 + r) * H + h) * dv + j0 + j] = acc[m];
                }
            }
        }
        __syncthreads();
        for (int c = tid; c < dk; c += kThreadsW) {
            gC[c] = g[((size_t)(t0 + L - 1) * H + h) * dk + c];
            gCl[c] = gl[((size_t)(t0 + L - 1) * H + h) * dk + c];
        }
        __syncthreads();
        for (int e = tid; e < L * dk; e += kThreadsW) {
            int r = e / dk, c = e - r * dk;
            size_t off = ((size_t)(t0 + r) * H + h) * dk + c;
            M[e] = to_f32(k[off]) * exp_gdiff(gC[c], gCl[c], g[off], gl[off]);
        }
        __syncthreads();
        // S <- Diag(exp(g_C)) S + (K . exp(g_C - g))^T W: thread t forms column t % 32
        // of rows t / 32 + 16 m (each element is read and written by its own thread)
        {
            const int j = tid & 31, c0 = tid >> 5;
            float acc[kMaxDK / 16];
#pragma unroll
            for (int m = 0; m < kMaxDK / 16; ++m) {
                const int c = c0 + 16 * m;
                acc[m] = c < dk ? exp_g(gC[c], gCl[c]) * S[c * kBV + j] : 0.f;
            }
            for (int r = 0; r < L; ++r) {
                const float w = Ws[r * kBV + j];
#pragma unroll
                for (int m = 0; m < kMaxDK / 16; ++m)
                    if (c0 + 16 * m < dk) acc[m] += M[r * dk + c0 + 16 * m] * w;
            }
#pragma unroll
            for (int m = 0; m < kMaxDK / 16; ++m) {
                const int c = c0 + 16 * m;
                if (c < dk) S[c * kBV + j] = acc[m];
            }
        }
        __syncthreads();
    }
    float* fdst = mcols ? map_out : final_state;
    if (fdst) {
        for (int e = tid; e < dk * kBV; e += kThreadsW) {
            int c = e / kBV, j = e - c * kBV;
            fdst[st_base + (size_t)c * ld + j0 + j] = S[e];
        }
    }
}

// K4: one block per (chunk, head).  Shared: Ks [C][dk] (then Q . exp(g)),
// Gs [C][dk], P [C][C], GLs [C][dk] (bf16, as in K2).
template <typename Tin>
__global__ void __launch_bounds__(kThreadsW) k4_output(const Tin* __restrict__ q, const Tin* __restrict__ k,
                                                      const float* __restrict__ g, const float* __restrict__ gl,
                                                      const float* __restrict__ Wg,
                                                      const float* __restrict__ S_chunk, Tin* __restrict__ o,
                                                      ChunkMap cmap, int H, int dk, int dv, int C) {
    extern __shared__ float smem[];
    int seq, tok0, len, idx;
    cmap.locate(blockIdx.x, seq, tok0, len, idx);
    const int h = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    float* Ks = smem;
    float* Gs = Ks + C * dk;
    float* P = Gs + C * dk;
    __nv_bfloat16* GLs = reinterpret_cast<__nv_bfloat16*>(P + C * C);
    for (int e = tid; e < len * dk; e += kThreadsW) {
        int r = e / dk, c = e - r * dk;
        size_t off = ((size_t)(tok0 + r) * H + h) * dk + c;
        Ks[e] = to_f32(k[off]);
        Gs[e] = g[off];
        GLs[e] = __float2bfloat16_rn(gl[off]);
    }
    __syncthreads();
    // P[r][i] = sum_c q_rc k_ic exp(g_rc - g_ic), i <= r (inclusive mask)
    for (int p = warp; p < len * len; p += kThreadsW / 32) {
        int r = p / len, i = p - r * len;
        float s = 0.f;
        if (i <= r) {
            const size_t qoff = ((size_t)(tok0 + r) * H + h) * dk;
            for (int c = lane; c < dk; c += 32)
                s += to_f32(q[qoff + c]) * Ks[i * dk + c] *
                     exp_gdiff(Gs[r * dk + c], __bfloat162float(GLs[r * dk + c]), Gs[i * dk + c],
                               __bfloat162float(GLs[i * dk + c]));
            s = warp_sum(s);
        }
        if (lane == 0) P[r * C + i] = s;
    }
    __syncthreads();
    for (int e = tid; e < len * dk; e += kThreadsW) {
        int r = e / dk, c = e - r * dk;
        size_t off = ((size_t)(tok0 + r) * H + h) * dk + c;
        Ks[e] = to_f32(q[off]) * exp_g(Gs[e], __bfloat162float(GLs[e]));
    }
    __syncthreads();
    const size_t sc_base = ((size_t)blockIdx.x * H + h) * dk * dv;
    for (int e = tid; e < len * dv; e += kThreadsW) {
        int r = e / dv, j = e - r * dv;
        float s = 0.f;
        for (int c = 0; c < dk; ++c) s += Ks[r * dk + c] * S_chunk[sc_base + (size_t)c * dv + j];
        for (int i = 0; i <= r; ++i) s += P[r * C + i] * Wg[((size_t)(tok0 + i) * H + h) * dv + j];
        o[((size_t)(tok0 + r) * H + h) * dv + j] = from_f32<Tin>(s);
    }
}

// K2's shared memory: A, then the larger of (Ks, Gs fp32 + GLs bf16) and X.
size_t k2_smem(int C, int dk, int dv) {
    const size_t phase1 = sizeof(float) * 2 * (size_t)C * dk + sizeof(__nv_bfloat16) * (size_t)C * dk;
    const size_t phase2 = sizeof(float) * (size_t)C * (dk + dv);
    return sizeof(float) * (size_t)C * C + (phase1 > phase2 ? phase1 : phase2);
}

template <typename Tin>
cudaError_t run(const Tin* q, const Tin* k, const Tin* v, const Tin* la, const Tin* beta, const float* init_state,
                Tin* o, float* final_state, const ChunkMap& cmap, const SeqMap& smap, int n_chunks, int n_seqs,
                int H, int dk, int dv, int C, const SimtWorkspace& ws, cudaStream_t stream) {
    const size_t smem2 = k2_smem(C, dk, dv);
    const size_t smem3 = sizeof(float) * ((size_t)dk * kBV + (size_t)C * dk + (size_t)C * kBV + 2 * dk);
    const size_t smem4 = sizeof(float) * (2 * (size_t)C * dk + (size_t)C * C) + sizeof(__nv_bfloat16) * (size_t)C * dk;
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(k2_wy<Tin>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem2))) return e;
    auto k3 = C == 128 ? k3_state<Tin, 128> : k3_state<Tin, 64>;
    if ((e = cudaFuncSetAttribute(k3, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem3))) return e;
    if ((e = cudaFuncSetAttribute(k4_output<Tin>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem4))) return e;
    if (n_chunks > 0) k1_cumsum<Tin><<<dim3(n_chunks, H), dk, 0, stream>>>(la, ws.g, ws.gl, cmap, H, dk);
    timing_mark(stream, 1);
    if (n_chunks > 0)
        k2_wy<Tin><<<dim3(n_chunks, H), kThreadsW, smem2, stream>>>(k, v, beta, ws.g, ws.gl, ws.U, ws.Wk, cmap, H, dk,
                                                                  dv, C);
    timing_mark(stream, 2);
    if (n_seqs > 0)
        k3<<<dim3(n_seqs, H, dv / kBV), kThreadsW, smem3, stream>>>(k, ws.g, ws.gl, ws.U, ws.Wk, ws.W, ws.S_chunk,
                                                                 init_state, final_state, smap, H, dk, dv, C,
                                                                 nullptr);
    timing_mark(stream, 3);
    if (n_chunks > 0)
        k4_output<Tin><<<dim3(n_chunks, H), kThreadsW, smem4, stream>>>(q, k, ws.g, ws.gl, ws.W, ws.S_chunk, o, cmap,
                                                                     H, dk, dv, C);
    timing_mark(stream, 4);
    return cudaGetLastError();
}

template <typename Tin>
cudaError_t run_states(const Tin* k, const Tin* v, const Tin* la, const Tin* beta, const float* init_state,
                       const ChunkMap& cmap, const SeqMap& smap, int n_chunks, int n_seqs, int H, int dk, int dv,
                       int C, const SimtWorkspace& ws, cudaStream_t stream) {
    const size_t smem2 = k2_smem(C, dk, dv);
    const size_t smem3 = sizeof(float) * ((size_t)dk * kBV + (size_t)C * dk + (size_t)C * kBV + 2 * dk);
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(k2_wy<Tin>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem2))) return e;
    auto k3 = C == 128 ? k3_state<Tin, 128> : k3_state<Tin, 64>;
    if ((e = cudaFuncSetAttribute(k3, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem3))) return e;
    if (n_chunks > 0) {
        k1_cumsum<Tin><<<dim3(n_chunks, H), dk, 0, stream>>>(la, ws.g, ws.gl, cmap, H, dk);
        k2_wy<Tin><<<dim3(n_chunks, H), kThreadsW, smem2, stream>>>(k, v, beta, ws.g, ws.gl, ws.U, ws.Wk, cmap, H, dk,
                                                                  dv, C);
    }
    if (n_seqs > 0)
        k3<<<dim3(n_seqs, H, dv / kBV), kThreadsW, smem3, stream>>>(k, ws.g, ws.gl, ws.U, ws.Wk, ws.W, ws.S_chunk,
                                                                 init_state, nullptr, smap, H, dk, dv, C, nullptr);
    return cudaGetLastError();
}

template <typename Tin>
cudaError_t run_map(const Tin* k, const Tin* v, const Tin* la, const Tin* beta, const ChunkMap& cmap,
                    const SeqMap& smap, int n_chunks, int n_seqs, int H, int dk, int dv, int C, const SimtWorkspace& ws,
                    float* Mmap, float* F, cudaStream_t stream) {
    const size_t smem2 = k2_smem(C, dk, dv);
    const size_t smem3 = sizeof(float) * ((size_t)dk * kBV + (size_t)C * dk + (size_t)C * kBV + 2 * dk);
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(k2_wy<Tin>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem2))) return e;
    auto k3 = C == 128 ? k3_state<Tin, 128, true> : k3_state<Tin, 64, true>;
    if ((e = cudaFuncSetAttribute(k3, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem3))) return e;
    if (n_chunks > 0) k1_cumsum<Tin><<<dim3(n_chunks, H), dk, 0, stream>>>(la, ws.g, ws.gl, cmap, H, dk);
    timing_mark(stream, 1);
    if (n_chunks > 0)
        k2_wy<Tin><<<dim3(n_chunks, H), kThreadsW, smem2, stream>>>(k, v, beta, ws.g, ws.gl, ws.U, ws.Wk, cmap, H, dk,
                                                                  dv, C);
    timing_mark(stream, 2);
    if (n_seqs > 0)
        k3<<<dim3(n_seqs, H, (dv + dk) / kBV), kThreadsW, smem3, stream>>>(k, ws.g, ws.gl, ws.U, ws.Wk, ws.W,
                                                                        ws.S_chunk, nullptr, F, smap, H, dk, dv, C,
                                                                        Mmap);
    timing_mark(stream, 3);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_simt_segment_map(kda_dtype dtype, const void* k, const void* v, const void* log_alpha,
                                    const void* beta, const ChunkMap& cmap, const SeqMap& smap, int n_chunks,
                                    int n_seqs, int H, int dk, int dv, int C, const SimtWorkspace& ws, float* Mmap,
                                    float* F, cudaStream_t stream) {
    if (dtype == KDA_F32)
        return run_map<float>((const float*)k, (const float*)v, (const float*)log_alpha, (const float*)beta, cmap,
                              smap, n_chunks, n_seqs, H, dk, dv, C, ws, Mmap, F, stream);
    return run_map<__nv_bfloat16>((const __nv_bfloat16*)k, (const __nv_bfloat16*)v, (const __nv_bfloat16*)log_alpha,
                                  (const __nv_bfloat16*)beta, cmap, smap, n_chunks, n_seqs, H, dk, dv, C, ws, Mmap, F,
                                  stream);
}

cudaError_t launch_simt_g(kda_dtype dtype, const void* log_alpha, const ChunkMap& cmap, int n_chunks, int H, int dk,
                          const SimtWorkspace& ws, cudaStream_t stream) {
    if (n_chunks == 0) return cudaSuccess;
    if (dtype == KDA_F32)
        k1_cumsum<float><<<dim3(n_chunks, H), dk, 0, stream>>>((const float*)log_alpha, ws.g, ws.gl, cmap, H, dk);
    else
        k1_cumsum<__nv_bfloat16><<<dim3(n_chunks, H), dk, 0, stream>>>((const __nv_bfloat16*)log_alpha, ws.g, ws.gl,
                                                                        cmap, H, dk);
    return cudaGetLastError();
}

cudaError_t launch_simt_states(kda_dtype dtype, const void* k, const void* v, const void* log_alpha,
                               const void* beta, const float* init_state, const ChunkMap& cmap, const SeqMap& smap,
                               int n_chunks, int n_seqs, int H, int dk, int dv, int C, const SimtWorkspace& ws,
                               cudaStream_t stream) {
    if (dtype == KDA_F32)
        return run_states<float>((const float*)k, (const float*)v, (const float*)log_alpha, (const float*)beta,
                                 init_state, cmap, smap, n_chunks, n_seqs, H, dk, dv, C, ws, stream);
    return run_states<__nv_bfloat16>((const __nv_bfloat16*)k, (const __nv_bfloat16*)v,
                                     (const __nv_bfloat16*)log_alpha, (const __nv_bfloat16*)beta, init_state, cmap,
                                     smap, n_chunks, n_seqs, H, dk, dv, C, ws, stream);
}

cudaError_t launch_simt_prefill(kda_dtype dtype, const void* q, const void* k, const void* v, const void* log_alpha,
                                const void* beta, const float* init_state, void* o, float* final_state,
                                const ChunkMap& cmap, const SeqMap& smap, int n_chunks, int n_seqs, int H, int dk,
                                int dv, int C, const SimtWorkspace& ws, cudaStream_t stream) {
    if (dtype == KDA_F32)
        return run<float>((const float*)q, (const float*)k, (const float*)v, (const float*)log_alpha,
                          (const float*)beta, init_state, (float*)o, final_state, cmap, smap, n_chunks, n_seqs, H,
                          dk, dv, C, ws, stream);
    return run<__nv_bfloat16>((const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v,
                              (const __nv_bfloat16*)log_alpha, (const __nv_bfloat16*)beta, init_state,
                              (__nv_bfloat16*)o, final_state, cmap, smap, n_chunks, n_seqs, H, dk, dv, C, ws, stream);
}

}  // namespace kda
