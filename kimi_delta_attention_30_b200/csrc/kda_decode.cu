// KDA decode step: one token per sequence, the fp32 state updated in place.
//
//   S~ = Diag(alpha) S            decay each key channel (row of S)
//   u  = v - S~^T k               error of the old answer read with the key
//   o  = S~^T q + beta (k . q) u  = S_new^T q
//   S  = S~ + beta k u^T          write the correction along the key
//
// Token-by-token decode (read state, emit output, update state): "我终于看懂了
// KDA" explainer (pwwt.cn/news/3787313), section 15; order decay -> read ->
// error -> write: same page, section 8; per-channel alpha: section 9.
//
// With kda_prep flags the kernel also normalises q and k, turns raw gate
// logits into log alpha = -softplus(a) and raw beta logits into sigmoid(b).
//
// The step is bound by HBM bandwidth: every state element is loaded once and
// stored once.  One 256-thread block owns one (sequence, head) state; a warp
// reads whole rows with 128-bit loads (coalesced), every thread keeps its
// slice of the state in registers between the read and the write, and the
// column sums S~^T k and S~^T q are reduced across warps through shared memory.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kThreads = 256;

template <typename Tin, int DK, int DV>
__global__ void __launch_bounds__(kThreads, 2)
decode_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
              const Tin* __restrict__ la, const Tin* __restrict__ beta, float* __restrict__ state,
              Tin* __restrict__ o, unsigned prep) {
    constexpr int V4 = DV / 4;          // float4 per state row
    constexpr int RPP = kThreads / V4;  // rows covered by one pass of the block
    constexpr int NR = DK / RPP;        // rows held by each thread
    static_assert(NR >= 1 && DK % RPP == 0, "tile");
    __shared__ float sk[DK], sq[DK], sa[DK], sv[DV], su[DV];
    __shared__ __align__(16) float red_r[RPP][DV];
    __shared__ __align__(16) float red_p[RPP][DV];
    __shared__ float s_kq, s_inv_k, s_inv_q;

    const int nh = blockIdx.x;
    const int tid = threadIdx.x, col4 = tid % V4, rg = tid / V4;
    float4* S4 = reinterpret_cast<float4*>(state + (size_t)nh * DK * DV);

    float4 s[NR];
#pragma unroll
    for (int i = 0; i < NR; ++i) s[i] = S4[(rg + i * RPP) * V4 + col4];

    for (int c = tid; c < DK; c += kThreads) {
        sk[c] = to_f32(k[(size_t)nh * DK + c]);
        sq[c] = to_f32(q[(size_t)nh * DK + c]);
        sa[c] = expf(prep_log_alpha(to_f32(la[(size_t)nh * DK + c]), prep));
    }
    for (int j = tid; j < DV; j += kThreads) sv[j] = to_f32(v[(size_t)nh * DV + j]);
    __syncthreads();

    // With the key/query normalisation the vectors stay raw: 1/||k|| and 1/||q|| scale
    // the reduced results (S^T k, S^T q, k.q) and the write, and come out of the same
    // warp-0 pass as k.q, so the normalisation adds no barrier.
    const bool l2 = (prep & KDA_PREP_QK_L2NORM) != 0;
    if (tid < 32) {
        float acc = 0.f, nk = 0.f, nq = 0.f;
        for (int c = tid; c < DK; c += 32) {
            acc += sk[c] * sq[c];
            if (l2) { nk += sk[c] * sk[c]; nq += sq[c] * sq[c]; }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            acc += __shfl_xor_sync(0xffffffffu, acc, off);
            if (l2) {
                nk += __shfl_xor_sync(0xffffffffu, nk, off);
                nq += __shfl_xor_sync(0xffffffffu, nq, off);
            }
        }
        if (tid == 0) {
            const float ik = l2 ? inv_norm_from_sq(nk) : 1.f, iq = l2 ? inv_norm_from_sq(nq) : 1.f;
            s_inv_k = ik;
            s_inv_q = iq;
            s_kq = acc * ik * iq;
        }
    }
    float4 racc = make_float4(0.f, 0.f, 0.f, 0.f), pacc = racc;
#pragma unroll
    for (int i = 0; i < NR; ++i) {
        const int c = rg + i * RPP;
        const float a = sa[c], kc = sk[c], qc = sq[c];
        s[i].x *= a; s[i].y *= a; s[i].z *= a; s[i].w *= a;
        racc.x += kc * s[i].x; racc.y += kc * s[i].y; racc.z += kc * s[i].z; racc.w += kc * s[i].w;
        pacc.x += qc * s[i].x; pacc.y += qc * s[i].y; pacc.z += qc * s[i].z; pacc.w += qc * s[i].w;
    }
    reinterpret_cast<float4*>(&red_r[rg][0])[col4] = racc;
    reinterpret_cast<float4*>(&red_p[rg][0])[col4] = pacc;
    __syncthreads();

    const float b = prep_beta(to_f32(beta[nh]), prep);
    const float ik = s_inv_k, iq = s_inv_q;
    for (int j = tid; j < DV; j += kThreads) {
        float r = 0.f, p = 0.f;
#pragma unroll
        for (int g = 0; g < RPP; ++g) { r += red_r[g][j]; p += red_p[g][j]; }
        r *= ik;
        p *= iq;
        const float u = sv[j] - r;
        su[j] = u;
        o[(size_t)nh * DV + j] = from_f32<Tin>(p + b * s_kq * u);
    }
    __syncthreads();

    const float4 u4 = reinterpret_cast<const float4*>(su)[col4];
#pragma unroll
    for (int i = 0; i < NR; ++i) {
        const float bk = b * ik * sk[rg + i * RPP];
        s[i].x += bk * u4.x; s[i].y += bk * u4.y; s[i].z += bk * u4.z; s[i].w += bk * u4.w;
        S4[(rg + i * RPP) * V4 + col4] = s[i];
    }
}

template <typename Tin>
cudaError_t run(const void* q, const void* k, const void* v, const void* la, const void* beta, float* state, int N,
                int H, int dk, int dv, void* o, unsigned prep, cudaStream_t stream) {
    const dim3 grid((unsigned)N * (unsigned)H);
    const Tin *Q = (const Tin*)q, *K = (const Tin*)k, *V = (const Tin*)v, *LA = (const Tin*)la, *BE = (const Tin*)beta;
    Tin* O = (Tin*)o;
    if (dk == 128 && dv == 128)
        decode_kernel<Tin, 128, 128><<<grid, kThreads, 0, stream>>>(Q, K, V, LA, BE, state, O, prep);
    else if (dk == 128 && dv == 64)
        decode_kernel<Tin, 128, 64><<<grid, kThreads, 0, stream>>>(Q, K, V, LA, BE, state, O, prep);
    else if (dk == 64 && dv == 128)
        decode_kernel<Tin, 64, 128><<<grid, kThreads, 0, stream>>>(Q, K, V, LA, BE, state, O, prep);
    else
        decode_kernel<Tin, 64, 64><<<grid, kThreads, 0, stream>>>(Q, K, V, LA, BE, state, O, prep);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(kda_dtype dtype, const void* q, const void* k, const void* v, const void* log_alpha,
                          const void* beta, float* state, int N, int H, int dk, int dv, void* o, unsigned prep,
                          cudaStream_t stream) {
    if (dtype == KDA_F32) return run<float>(q, k, v, log_alpha, beta, state, N, H, dk, dv, o, prep, stream);
    return run<__nv_bfloat16>(q, k, v, log_alpha, beta, state, N, H, dk, dv, o, prep, stream);
}

}  // namespace kda
